// gdn_internal.cuh -- argument blocks and launcher declarations shared by the C-ABI layer
// (gdn_abi.cu) and the kernel translation units. Not part of the public interface.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace gdn {

// Streaming multiprocessors of the current device, asked of the runtime once per device.
inline cudaError_t current_sm_count(int* nsm) {
    static std::atomic<int> cache[64];   // 0: not asked yet
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) {
            *nsm = c;
            return cudaSuccess;
        }
    }
    e = cudaDeviceGetAttribute(nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess && dev >= 0 && dev < 64) cache[dev].store(*nsm, std::memory_order_relaxed);
    return e;
}

// The dynamic shared memory a kernel may use, set once per (kernel, device): the attribute
// belongs to the function on the current device.
template <auto Kernel>
inline cudaError_t ensure_smem_attr(int bytes) {
    static std::atomic<uint64_t> done{0};   // bit d: set on device d
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t{1} << dev) : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// Arguments of one verify / decode launch (layouts as in include/gdn.h).
struct VerifyArgs {
    int B, T, Hk, Hv, dk, dv;
    int in_bf16, out_bf16;
    const void* q;
    const void* k;
    const void* v;
    const void* a;
    const void* b;
    const float* A_log;
    const float* dt_bias;
    const float* state_in;
    float* state_out;
    const int32_t* accept_len;   // NULL: no fused commit (two-phase or decode)
    void* o;
    float* stash;                // NULL: no stash
    float l2_eps, scale;
    int32_t* status_word;
    int always_commit;           // decode: commit all T tokens, ignore accept_len
    int row_split;               // head kernel: CTAs (work items) per head, set by its launcher
    int prefetch_ahead;          // tensor-core verify: the item whose inputs a CTA prefetches into
                                 // L2 is its own + this (0: none), set by its launcher
    // Commit-on-next-verify (tensor-core kernel only): the previous two-phase block's stash
    // (prev_T tokens) and accept counts, applied to state_in before this block (NULL: none).
    const float* prev_stash;
    const int32_t* prev_accept_len;
    int prev_T;
    // Gated RMS normalisation of the outputs (NULL norm_z: none): o <- o / sqrt(mean(o^2) + eps)
    // * norm_w * silu(norm_z) per (token, value head); norm_z has v's layout and dtype.
    const void* norm_z;
    const float* norm_w;
    float norm_eps;
    // Programmatic dependent launch (GDN_LAUNCH_PDL): honoured by the one-CTA-per-head kernel.
    int pdl;
};

// Arguments of the second phase of a two-phase commit.
struct CommitArgs {
    int B, T, Hv, dk, dv;
    const float* state_in;
    float* state_out;
    const float* stash;
    const int32_t* accept_len;
    int32_t* status_word;
};

// Stash of one (sequence, value head), in floats: khat [T][d_k], cumulative log-decay
// G [T] padded to a multiple of 4, then u [T][d_v] padded to a multiple of 4. Every part
// starts on a 16-byte boundary.
__host__ __device__ inline size_t stash_floats_per_head(int T, int dk, int dv) {
    return (size_t)T * dk + (((size_t)T + 3) & ~size_t(3)) + (((size_t)T * dv + 3) & ~size_t(3));
}

// Causal short convolution over q | k | v with its rewound history (gdn_conv.cu).
struct ConvArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* w;              // [C][K] fp32
    const void* hist_in;         // [B][K-1][C] in_dtype
    void* hist_out;              // [B][K-1][C] in_dtype, or nullptr (history not written)
    const int32_t* accept_len;   // [B] device, or nullptr (all T accepted)
    void* q_out;                 // post-convolution q, k, v (in_dtype), or all nullptr
    void* k_out;
    void* v_out;
    int32_t* status_word;
    int B, T, C, Cq;             // C = 2 Cq + H_v d_v channels, Cq = H_k d_k
    int tile;                    // tokens per thread (set by the launcher)
    bool fused_hist;             // this launch also rewinds the history (set by the launcher)
};

// Host launchers; return cudaSuccess or the launch error. Shapes are validated by the caller.
cudaError_t launch_verify(const VerifyArgs& a, cudaStream_t stream);
// Name of the kernel the calling thread's last launch_verify chose ("" before the first).
const char* last_verify_kernel();
cudaError_t launch_short_conv(const ConvArgs& a, int K, bool bf16, cudaStream_t stream);

// Gated RMS normalisation of rows of d elements (gdn_norm.cu). y may be x (in place).
struct NormArgs {
    const void* x;       // [rows][d], fp32 or bf16
    const void* z;       // [rows][d], fp32 or bf16
    const float* w;      // [d]
    void* y;             // [rows][d], fp32 or bf16
    int64_t rows;
    int d;               // a multiple of 4, <= 4096
    float eps;
    bool x_bf16, z_bf16, y_bf16;
};
cudaError_t launch_gated_rmsnorm(const NormArgs& a, cudaStream_t stream);

// Device-side acceptance of a verify block (gdn_accept.cu).
struct AcceptRowStat {
    float m;     // greedy: the row's maximum logit; sampled: max of logit log2(e) / tau
    float s;     // sampled: sum of 2^(logit log2(e) / tau - m)
    int arg;     // greedy: first index of the maximum
    int pad;
};
struct AcceptArgs {
    int B, T, V;
    bool bf16, sampled;
    float tau;
    const void* target;          // [B][T][V]
    const void* draft;           // [B][T-1][V] (sampled)
    const int32_t* tokens;       // [B][T]: the anchor, then the drafts
    const float* u;              // [B][T] (sampled): u[0] for the draw, u[t+1] for draft t+1
    int32_t* accept_len;         // [B] out
    int32_t* next_token;         // [B] out
    int32_t* status_word;
    // Set by the launcher from the workspace:
    AcceptRowStat* stats;        // row statistics
    int* nsurv;                  // surviving drafts per sequence
    int* counters;               // [2 B]: rows done per sequence, draw CTAs done per sequence
    int* decided;                // [B] 1 once the sequence's counts are written (zeroed with
                                 //     the counters)
    uint32_t max_polls;          // bound of a draw CTA's wait for its flag (0: the default)
    float* tiles;                // residual tile sums per sequence
};
size_t accept_workspace_bytes(int B, int T, int V, bool sampled);

// A bounded wait that nothing completes (gdn_selftest.cu).
cudaError_t launch_bounded_wait_selftest(int32_t* status_word, uint32_t polls, cudaStream_t stream);
cudaError_t launch_accept(AcceptArgs a, void* workspace, cudaStream_t stream);
// The acceptance draw kernel alone, waiting `polls` polls on a flag that nothing raises.
cudaError_t launch_accept_wait_selftest(int32_t* status_word, int32_t* next_token, uint32_t polls,
                                        cudaStream_t stream);

// One CTA per (sequence, value head) form for d_k = 128, d_v <= 128, T <= 16.
bool head_kernel_applies(const VerifyArgs& a);

// Latency form for fewer (sequence, value head) pairs than SMs: the per-token recurrence on
// 16-row state slices in registers (d_k = 128, d_v a multiple of 16, T <= 16, fused commit or
// decode, no stash).
bool rec_kernel_applies(const VerifyArgs& a, int num_sms);
cudaError_t launch_verify_rec(const VerifyArgs& a, cudaStream_t stream);

// Tensor-core form (d_k = d_v = 128, T <= 8, at least one (sequence, head) per SM).
bool tc_kernel_applies(const VerifyArgs& a, int num_sms);
cudaError_t launch_verify_tc(const VerifyArgs& a, cudaStream_t stream);
// Persistent warp-specialised tensor-core form: the same shapes, with the commit fused at
// device accept counts (no stash, no previous-block commit, no gated norm).
bool pipe_kernel_applies(const VerifyArgs& a, int num_sms);
cudaError_t launch_verify_pipe(const VerifyArgs& a, cudaStream_t stream);
cudaError_t launch_verify_head(const VerifyArgs& a, cudaStream_t stream);
cudaError_t launch_commit(const CommitArgs& a, cudaStream_t stream);

}  // namespace gdn
