// gdn_prefill.cu -- long-prompt prefill of the Gated DeltaNet mixer on tcgen05 tensor cores.
//
// The chunked form of the recurrence (chunk C = 64; the same block algebra as the verify
// kernels, taken one chunk at a time): for a chunk with state S at its start, G_t the
// chunk-local inclusive cumulative log-decay, d_t = exp(G_t), d_C = d_{C-1},
//   Gram:   Kk = Khat Khat^T, Qk = Qhat Khat^T                      (64 x 64 each)
//   A[t][s] = beta_t exp(G_t - G_s) Kk[t][s] (s < t),  Tm = (I + A)^-1
//   Cq[t][s] = exp(G_t - G_s) Qk[t][s] (s <= t),      Mo = Cq Tm
//   Keff_s = sum_{t >= s} exp(G_C - G_t) Tm[t][s] khat_t              (folded keys)
//   P | R  = S [Khat; Qhat]^T                                          (128 x 128)
//   X[i][s] = beta_s (v_s[i] - d_s P[i][s])
//   O[i][t] = d_t R[i][t] + (X Mo^T)[i][t]
//   S      <- d_C S + X Keff
// Two kernels, run over a long prompt in up to four pieces of whole chunks, the scan of one
// piece beside the preparation of the next (launch_prefill):
//   gdn_prefill_prep_kernel, one CTA per (sequence, key head, chunk), all in parallel: the
//     state-independent part. Normalised keys / queries and their Gram matrix (tensor cores),
//     once for all value heads of the group; per value head, the gates and
//     then Mo and Keff^T without forming Tm: both solve x (I + A) = y for a row vector y (a row
//     of Cq, or the column exp(G_C - G_t) khat_t[j] for one key dimension j), which one thread
//     does by right-looking back substitution in registers. The results go to the workspace in
//     the exact shared-memory image the scan consumes (the scan copies them in whole).
//   gdn_prefill_scan_kernel, one CTA per (sequence, value head), chunk after chunk (over a
//     range of chunks, from the state the previous range left), warp
//     specialised: warp 8 streams the chunk operands in (bulk copies and a TMA tensor copy of
//     V) and issues the tensor-core MMAs; warps 0-7 form X and write the outputs. The state
//     lives in tensor memory (fp32) as the A operand of P | R and the accumulator of the
//     update. Two wide MMA chains per chunk ([P | R], N = 128; [O | S update], N = 192): the
//     tf32 MMA has a large fixed cost per instruction, so fewer, wider ones finish sooner. Its per-chunk decay d_C is carried in a scalar sigma (state = sigma * S~) and
//     folded into X, so the tensor-memory state is only rescaled when sigma would fall below
//     2^-32.
// Precision (kind::tf32 reads operands as truncated tf32): S [Khat; Qhat]^T and the Gram take
// one tf32 pass; X Mo^T and X Keff take two (X split into a tf32 high part and the fp32
// remainder, against Mo / Keff^T rounded to the nearest tf32 by the prep kernel). An fp32
// emulation of exactly this arithmetic against the fp64 recurrence gives ~8e-4 relative error
// in o and ~2e-4 in the state at worst.
// Every mbarrier wait is bounded; a timeout sets GDN_STATUS_WAIT_TIMEOUT, every thread of the
// CTA stops, the CTA waits (bounded) for the copies and MMAs it issued and frees its tensor
// memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "gdn_device.cuh"
#include "gdn_internal.cuh"
#include "gdn_prefill.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {
using namespace dev;

constexpr int kC = 64;                  // chunk length
constexpr int DK = 128;
constexpr int DV = 128;
constexpr int kPrepThreads = 256;
constexpr int kScanThreads = 288;       // warps 0-7 form X / outputs, warp 8 loads and issues MMAs
constexpr uint32_t kMaxPolls = 1u << 24;

// Workspace, two arrays:
//   KQ tiles, one per (sequence, key head, chunk): [khat; qhat] (128 rows x 128 fp32) in the
//     K-major SWIZZLE_128B image (four 32-column blocks of [128 rows][32]).
//   Records, one per (sequence, value head, chunk):
//     B2  [192 rows][64 s] K-major SWIZZLE_128B image (two blocks of [192][32]):
//         rows 0..63 Mo (row t = Mo[t][s]), rows 64..191 Keff^T (row j = Keff_s[j] over s);
//         values rounded to the nearest tf32. One N = 192 MMA against it gives [O | S update].
//     vec d[64] | beta[64] | d_C | pad  (144 fp32)
constexpr int kRecRows = DK + kC;                             // 192
constexpr uint32_t kKQBytes = 2 * kC * DK * 4;                // 65536
constexpr uint32_t kB2Bytes = kRecRows * kC * 4;              // 49152
constexpr uint32_t kVecFloats = 144;
constexpr uint32_t kRecBytes = kB2Bytes + kVecFloats * 4;     // 49728
constexpr uint32_t kKBlock = 2 * kC * 128;                    // bytes per 32-column block of a KQ tile
constexpr uint32_t kRBlock = kRecRows * 128;                  // bytes per 32-column block of B2

__host__ __device__ inline size_t n_chunks_of(int T) { return ((size_t)T + kC - 1) / kC; }

// ---------------------------------------------------------------- prep kernel

constexpr int kApad = 68;               // A row stride (floats): 16-byte rows, float4 stores conflict-free
constexpr float kLog2e = 1.4426950408889634f;

// One CTA per (sequence, key head, chunk): keys / queries, their normalisation and Gram matrix
// are the same for every value head of the group; gates, decays and the solves are per value
// head. A and the gate vectors are double-buffered so that warps 0, 1 prepare the next value
// head while warps 2-7 solve the current one.
struct __align__(1024) PrepSmem {
    float KQ[2 * kC * DK];     // [khat; qhat] SW128 image (Gram operands, Keff right-hand sides)
    float A[2][kC][kApad];     // strictly lower A
    float G2[2][kC];           // inclusive cumulative log2-decay over the chunk
    float Beta[2][kC];
    float Ec[2][kC];           // 2^(G2_{n-1} - G2_t)
    uint64_t mma_done;
    uint32_t tmem;
};

// x (I + A) = y for the row vector x, A strictly lower triangular (shared memory, row m holds
// A[m][0..m)), y given in acc and overwritten by x. Right-looking back substitution: x_m is
// final once every x_{m'} with m' > m has been subtracted out, then x_m A[m][s] is removed from
// every s < m. A[m][s] = 0 for s >= m, so whole float4 groups of row m can be used.
__device__ __forceinline__ void solve_unit_lower_row(float2 (&acc)[kC / 2], const float (*A)[kApad]) {
#pragma unroll
    for (int m = kC - 1; m > 0; --m) {
        const float xm = (m & 1) ? acc[m >> 1].y : acc[m >> 1].x;
        const float2 nx = make_float2(-xm, -xm);
#pragma unroll
        for (int f = 0; f < (m + 3) / 4; ++f) {
            const float4 a = *reinterpret_cast<const float4*>(&A[m][4 * f]);
            acc[2 * f] = __ffma2_rn(nx, make_float2(a.x, a.y), acc[2 * f]);
            if (2 * f + 1 < kC / 2) acc[2 * f + 1] = __ffma2_rn(nx, make_float2(a.z, a.w), acc[2 * f + 1]);
        }
    }
}

// Warps 0, 1 (token t = threadIdx.x): the gates of value head h over this chunk into buffer
// buf (log2 units), and the record's vec (d_t, beta_t, d_C). Named barrier 1 orders the two
// warps' halves of the prefix sum.
template <typename InT>
__device__ __forceinline__ void prep_head_gates(const VerifyArgs& p, PrepSmem& sm, int buf, int b, int h, int t0,
                                                int n, float* vec) {
    const int t = threadIdx.x;
    const int lane = t & 31;
    float gl = 0.f, be = 0.f;
    if (t < n) {
        const size_t gi = ((size_t)b * p.T + t0 + t) * p.Hv + h;
        gl = -expf(p.A_log[h]) * softplus_f(ld_in<InT>(p.a, gi) + p.dt_bias[h]) * kLog2e;
        be = 1.f / (1.f + expf(-ld_in<InT>(p.b, gi)));
    }
    float Gs = gl;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(kFull, Gs, off);
        if (lane >= off) Gs += y;
    }
    sm.G2[buf][t] = Gs;
    sm.Beta[buf][t] = be;
    named_barrier_sync(1, 2 * 32);
    if (t >= 32) sm.G2[buf][t] = Gs + sm.G2[buf][31];
    named_barrier_sync(1, 2 * 32);
    const float GC = sm.G2[buf][n - 1];
    const float G = sm.G2[buf][t];
    sm.Ec[buf][t] = t < n ? exp2_approx(GC - G) : 0.f;
    vec[t] = t < n ? exp2_approx(G) : 0.f;
    vec[kC + t] = be;
    if (t == 0) vec[2 * kC] = exp2_approx(GC);
    named_barrier_sync(1, 2 * 32);
}

// Warps 0, 1 (row t = threadIdx.x): A[t][s] = beta_t 2^(G2_t - G2_s) Kk[t][s] for s < t, from
// Gram row t in tensor memory, into A[buf].
__device__ __forceinline__ void prep_rows_A(PrepSmem& sm, int buf, uint32_t tmem, int n) {
    const int t = threadIdx.x;
    float gv[kC];
#pragma unroll
    for (int cb = 0; cb < kC; cb += 16)
        tc::tmem_ld16(tmem + ((uint32_t)(t & ~31) << 16) + cb, *reinterpret_cast<float(*)[16]>(&gv[cb]));
    const float Gt = sm.G2[buf][t], bt = sm.Beta[buf][t];
#pragma unroll
    for (int s4 = 0; s4 < kC; s4 += 4) {
        float a[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int s = s4 + e;
            a[e] = (s < t && t < n) ? bt * exp2_approx(Gt - sm.G2[buf][s]) * gv[s] : 0.f;
        }
        *reinterpret_cast<float4*>(&sm.A[buf][t][s4]) = make_float4(a[0], a[1], a[2], a[3]);
    }
}

// Warps 2-7, the right-hand sides of the solves for the value head in buffer buf. Warps 2, 3
// (Mo row t = tid - 64): Cq[t][s] = 2^(G2_t - G2_s) Qk[t][s], s <= t, from Gram row 64 + t.
// Warps 4-7 (key dimension j = tid - 128): Ec_s khat_s[j].
__device__ __forceinline__ void prep_rhs(const PrepSmem& sm, int buf, uint32_t tmem, int n, float2 (&acc)[kC / 2]) {
    const int tid = threadIdx.x;
    if (tid < 128) {
        float gv[kC];
#pragma unroll
        for (int cb = 0; cb < kC; cb += 16)
            tc::tmem_ld16(tmem + ((uint32_t)(tid & ~31) << 16) + cb, *reinterpret_cast<float(*)[16]>(&gv[cb]));
        const int t = tid - kC;
        const float Gt = sm.G2[buf][t];
#pragma unroll
        for (int s2 = 0; s2 < kC / 2; ++s2) {
            const int s = 2 * s2;
            acc[s2].x = (s <= t && t < n) ? exp2_approx(Gt - sm.G2[buf][s]) * gv[s] : 0.f;
            acc[s2].y = (s + 1 <= t && t < n) ? exp2_approx(Gt - sm.G2[buf][s + 1]) * gv[s + 1] : 0.f;
        }
    } else {
        const int j = tid - 128;
#pragma unroll
        for (int s2 = 0; s2 < kC / 2; ++s2) {
            const int s = 2 * s2;
            acc[s2].x = sm.Ec[buf][s] * sm.KQ[tc::sw128_offset(s, j, 2 * kC) / 4];
            acc[s2].y = sm.Ec[buf][s + 1] * sm.KQ[tc::sw128_offset(s + 1, j, 2 * kC) / 4];
        }
    }
}

template <typename InT>
__global__ void __launch_bounds__(kPrepThreads, 2)
    gdn_prefill_prep_kernel(const VerifyArgs p, float* __restrict__ ws_kq, unsigned char* __restrict__ ws_rec,
                            int c_first) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    PrepSmem& sm = *reinterpret_cast<PrepSmem*>(smem_raw);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int c = c_first + (int)blockIdx.x;
    const int g = blockIdx.y;
    const int b = blockIdx.z;
    const int T = p.T;
    const int grp = p.Hv / p.Hk;
    const size_t nch = n_chunks_of(T);
    const int t0 = c * kC;
    const int n = min(kC, T - t0);   // tokens in this chunk
    auto record = [&](int hh) { return ws_rec + (((size_t)b * p.Hv + (size_t)g * grp + hh) * nch + c) * kRecBytes; };

    if ((smem_u32(smem_raw) & 1023u) != 0) {
        if (tid == 0 && p.status_word) atomicOr(p.status_word, kStatusWaitTimeout);
        return;
    }
    if (tid == 0) {
        mbar_init(&sm.mma_done, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(&sm.tmem, 64);
        tc::tmem_relinquish();
    }

    // 1. Gates of the group's first value head (warps 0, 1), then the khat / qhat rows: 16
    // threads x 8 columns per row, 16 rows per pass, all loads in flight; written to shared
    // memory and, as the same SW128 image, to the workspace for the scan.
    if (warp < 2) prep_head_gates<InT>(p, sm, 0, b, g * grp, t0, n, reinterpret_cast<float*>(record(0) + kB2Bytes));
    {
        float* kq_dst = ws_kq + (((size_t)b * p.Hk + g) * nch + c) * (kKQBytes / 4);
        const int c16 = tid & 15;
        float x[8][8];
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int r = 16 * it + (tid >> 4);   // rows 0..63 khat, 64..127 qhat
            const bool isq = r >= kC;
            const int t = isq ? r - kC : r;
            if (t < n) {
                ld8<InT>(isq ? p.q : p.k, (((size_t)b * T + t0 + t) * p.Hk + g) * DK + 8 * c16, x[it]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[it][e] = 0.f;
            }
        }
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int r = 16 * it + (tid >> 4);
            const bool isq = r >= kC;
            const int t = isq ? r - kC : r;
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(x[it][e], x[it][e], ss);
            ss = group_sum<16>(ss);
            const float inv = t < n ? (isq ? p.scale : 1.f) / sqrtf(ss + p.l2_eps) : 0.f;
            const float4 lo = make_float4(x[it][0] * inv, x[it][1] * inv, x[it][2] * inv, x[it][3] * inv);
            const float4 hi = make_float4(x[it][4] * inv, x[it][5] * inv, x[it][6] * inv, x[it][7] * inv);
            const uint32_t o0 = tc::sw128_offset(r, 8 * c16, 2 * kC) / 4;
            const uint32_t o1 = tc::sw128_offset(r, 8 * c16 + 4, 2 * kC) / 4;
            *reinterpret_cast<float4*>(&sm.KQ[o0]) = lo;
            *reinterpret_cast<float4*>(&sm.KQ[o1]) = hi;
            *reinterpret_cast<float4*>(&kq_dst[o0]) = lo;
            *reinterpret_cast<float4*>(&kq_dst[o1]) = hi;
        }
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem;

    // 2. Gram on the tensor cores: D (128 x 64) = [Khat; Qhat] Khat^T, one tf32 pass. It stays
    // in tensor memory for every value head of the group.
    if (tid == 0) {
        const uint32_t id = tc::idesc_tf32(2 * kC, kC);
        const uint32_t kq = smem_u32(sm.KQ);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint32_t off = kb * kKBlock + ks * 32;
                tc::mma_tf32_ss(tmem, tc::desc_kmajor_sw128(kq + off), tc::desc_kmajor_sw128(kq + off), id,
                                kb + ks > 0);
            }
        tc::mma_commit(&sm.mma_done);
    }
    const bool ok = mbar_wait_bounded(&sm.mma_done, 0, kMaxPolls);
    tc::fence_after_sync();
    if (warp < 2) prep_rows_A(sm, 0, tmem, n);
    tc::fence_before_sync();
    __syncthreads();

    // 3. Per value head hh: warps 2-7 solve (warps 2, 3 give Mo rows 0..63, warps 4-7 Keff^T
    // rows 64..191) and write the rows, rounded to tf32, straight into the record's B2 image;
    // meanwhile warps 0, 1 prepare head hh + 1.
    for (int hh = 0; hh < grp; ++hh) {
        const int buf = hh & 1;
        if (warp >= 2) {
            float2 acc[kC / 2];
            prep_rhs(sm, buf, tmem, n, acc);
            if (ok) {
                solve_unit_lower_row(acc, sm.A[buf]);
                const int row = warp < 4 ? tid - 64 : kC + (tid - 128);
                float* rec = reinterpret_cast<float*>(record(hh));
#pragma unroll
                for (int f = 0; f < kC / 4; ++f) {
                    const float4 v = make_float4(tc::tf32_rna(acc[2 * f].x), tc::tf32_rna(acc[2 * f].y),
                                                 tc::tf32_rna(acc[2 * f + 1].x), tc::tf32_rna(acc[2 * f + 1].y));
                    *reinterpret_cast<float4*>(&rec[tc::sw128_offset(row, 4 * f, kRecRows) / 4]) = v;
                }
            }
        } else if (hh + 1 < grp) {
            prep_head_gates<InT>(p, sm, buf ^ 1, b, g * grp + hh + 1, t0, n,
                                 reinterpret_cast<float*>(record(hh + 1) + kB2Bytes));
            prep_rows_A(sm, buf ^ 1, tmem, n);
        }
        tc::fence_before_sync();
        __syncthreads();
    }
    if (!ok && tid == 0 && p.status_word) atomicOr(p.status_word, kStatusWaitTimeout);
    if (warp == 0) tc::tmem_dealloc(tmem, 64);
}

// ---------------------------------------------------------------- scan kernel

// Dynamic shared memory (byte offsets): the KQ tile, two record buffers, two V tiles; the
// barriers sit in the slack after record buffer 0.
constexpr uint32_t kOffKQ = 0;
constexpr uint32_t kRecStride = 50176;                  // kRecBytes rounded up to 1024
constexpr uint32_t kOffRec0 = kKQBytes;
constexpr uint32_t kOffRec1 = kOffRec0 + kRecStride;
constexpr uint32_t kOffBar = kOffRec0 + kRecBytes;
constexpr uint32_t kOffV0 = kOffRec1 + kRecStride;
template <typename InT>
__host__ __device__ constexpr uint32_t v_tile_bytes() { return kC * DV * sizeof(InT); }
template <typename InT>
__host__ __device__ constexpr uint32_t scan_smem_bytes() { return kOffV0 + 2 * v_tile_bytes<InT>(); }

struct ScanBars {
    uint64_t kq_full, rec_full[2], v_full[2];
    uint64_t mma_pr, mma_so, drain;
    uint64_t x_ready, o_free;           // 256 arrivals each
    uint32_t tmem;
    int abort;
};
static_assert(kOffBar + sizeof(ScanBars) <= kOffRec1, "barriers overflow the record slack");

// TMEM columns: [O | S~] 0..191 (one N = 192 accumulator: O 0..63, S~ 64..191), [P | R]
// 256..383, X_hi 384..447, X_lo 448..511 (each accumulator starts at a multiple of its width).
constexpr uint32_t kColO = 0, kColS = 64, kColPR = 256, kColXh = 384, kColXl = 448;
constexpr float kRenormBelow = 2.3283064365386963e-10f;   // 2^-32

// Bounded wait that also gives up once another thread of the CTA has given up.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort) {
    for (uint32_t i = 0; i < kMaxPolls; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *abort) return false;
    }
    *abort = 1;
    return false;
}

// D (+)= A B over K = 32 nkb: A from tensor memory (columns a0 + 32 kb + 8 ks), B from the
// K-major SW128 tile whose descriptor is b0 (32-column blocks kb_bytes apart; the start
// address field advances by bytes / 16, which stays inside its 14 bits for shared addresses).
// The first MMA overwrites D unless accumulate is set.
__device__ __forceinline__ void mma_ts_k(uint32_t d, uint32_t a0, uint64_t b0, uint32_t kb_bytes, int nkb,
                                         uint32_t idesc, bool accumulate) {
#pragma unroll 1
    for (int kb = 0; kb < nkb; ++kb) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            tc::mma_tf32_ts(d, a0 + kb * 32 + ks * 8, b0 + ((kb * kb_bytes + ks * 32) >> 4), idesc,
                            accumulate || kb + ks > 0);
    }
}

// The decay bookkeeping shared by producer and consumers (identical fp32 arithmetic on both
// sides): sigma_next = sigma d_C; below 2^-32 (or not a number) the decay is folded into S~
// instead and sigma restarts at 1.
__device__ __forceinline__ bool decay_renorm(float snext) { return !(snext >= kRenormBelow); }

template <typename InT, typename OutT>
__global__ void __launch_bounds__(kScanThreads, 1)
    gdn_prefill_scan_kernel(const __grid_constant__ CUtensorMap v_map, const VerifyArgs p,
                            const float* __restrict__ ws_kq, const unsigned char* __restrict__ ws_rec,
                            int c_begin, int c_end) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    constexpr uint32_t kVBytes = v_tile_bytes<InT>();
    ScanBars& bar = *reinterpret_cast<ScanBars*>(smem_raw + kOffBar);
    float* KQ = reinterpret_cast<float*>(smem_raw + kOffKQ);
    // Record buffer i at kOffRec0 + i * kRecStride, V buffer i at kOffV0 + i * kVBytes.
    auto REC = [&](int i) { return smem_raw + kOffRec0 + (uint32_t)i * kRecStride; };
    auto VT = [&](int i) { return smem_raw + kOffV0 + (uint32_t)i * kVBytes; };
    volatile int* abort = &bar.abort;

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int h = blockIdx.x;
    const int b = blockIdx.y;
    const int T = p.T;
    const int grp = p.Hv / p.Hk;
    const int g = h / grp;
    const int nch = (int)n_chunks_of(T);
    const size_t head = (size_t)b * p.Hv + h;
    const float* kq_src = ws_kq + ((size_t)b * p.Hk + g) * nch * (kKQBytes / 4);
    const unsigned char* rec_src = ws_rec + head * nch * kRecBytes;

    if ((smem_u32(smem_raw) & 1023u) != 0) {
        if (tid == 0 && p.status_word) atomicOr(p.status_word, kStatusWaitTimeout);
        return;
    }
    if (tid == 0) {
        mbar_init(&bar.kq_full, 1);
        mbar_init(&bar.rec_full[0], 1);
        mbar_init(&bar.rec_full[1], 1);
        mbar_init(&bar.v_full[0], 1);
        mbar_init(&bar.v_full[1], 1);
        mbar_init(&bar.mma_pr, 1);
        mbar_init(&bar.mma_so, 1);
        mbar_init(&bar.drain, 1);
        mbar_init(&bar.x_ready, 256);
        mbar_init(&bar.o_free, 256);
        bar.abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(&bar.tmem, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = bar.tmem;

    // Loads issued by the producer thread, counted per barrier for the drain.
    uint32_t n_kq = 0, n_rec0 = 0, n_rec1 = 0, n_v0 = 0, n_v1 = 0;
    const bool producer = tid == 256;
    auto load_kq = [&](int c) {
        mbar_arrive_expect_tx(&bar.kq_full, kKQBytes);
        bulk_g2s(KQ, kq_src + (size_t)c * (kKQBytes / 4), kKQBytes, &bar.kq_full);
        ++n_kq;
    };
    // Buffers and barrier phases follow the chunk's place in this launch's range, c - c_begin.
    auto load_rec = [&](int c) {
        const int s = (c - c_begin) & 1;
        mbar_arrive_expect_tx(&bar.rec_full[s], kRecBytes);
        bulk_g2s(REC(s), rec_src + (size_t)c * kRecBytes, kRecBytes, &bar.rec_full[s]);
        if (s) ++n_rec1; else ++n_rec0;
    };
    auto load_v = [&](int c) {
        const int s = (c - c_begin) & 1;
        mbar_arrive_expect_tx(&bar.v_full[s], kVBytes);
        tc::tma_load_4d(VT(s), &v_map, 0, h, c * kC, b, &bar.v_full[s]);
        if (s) ++n_v1; else ++n_v0;
    };
    if (producer) {
        load_kq(c_begin);
        load_rec(c_begin);
        load_v(c_begin);
        if (c_end - c_begin > 1) {
            load_rec(c_begin + 1);
            load_v(c_begin + 1);
        }
    }

    // Consumer geometry: warp w owns TMEM lanes 32 (w % 4) .. +31 (state rows) and token
    // columns 32 (w / 4) .. +31 of each chunk.
    const int q4 = warp & 3;
    const int half = (warp >> 2) & 1;
    const int row = 32 * q4 + lane;
    const uint32_t lb = tmem + ((uint32_t)(32 * q4) << 16);

    // Initial state (zero when state_in is NULL) into tensor memory, columns 64 half .. +63 of
    // S~, and zeros in this thread's O columns.
    if (warp < 8) {
        const float* src = p.state_in ? p.state_in + (head * DV + row) * DK + 64 * half : nullptr;
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) {
            float v[32];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 x = src ? __ldg(reinterpret_cast<const float4*>(src + 32 * cb) + q)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                v[4 * q] = x.x;
                v[4 * q + 1] = x.y;
                v[4 * q + 2] = x.z;
                v[4 * q + 3] = x.w;
            }
            tc::tmem_st32(lb + kColS + 64 * half + 32 * cb, v);
        }
        float z[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) z[e] = 0.f;
        tc::tmem_st32(lb + kColO + 32 * half, z);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();

    bool ok = true;
    if (producer) {
        // ---------------- producer / MMA issuer
        const uint32_t idPR = tc::idesc_tf32(DV, 2 * kC), idSO = tc::idesc_tf32(DV, kRecRows);
        const uint64_t dKQ = tc::desc_kmajor_sw128(smem_u32(KQ));
        float sigma = 1.f;   // mirrors the consumers' decay scalar
        for (int c = c_begin; c < c_end; ++c) {
            const int i = c - c_begin;
            if (!wait_or_abort(&bar.kq_full, i & 1, abort)) { ok = false; break; }
            // S~ is final once the previous update is done.
            if (i >= 1 && !wait_or_abort(&bar.mma_so, (i - 1) & 1, abort)) { ok = false; break; }
            tc::fence_after_sync();
            // [P | R]_c = S~ [Khat; Qhat]^T (A = S~ in tensor memory, one pass, N = 128).
            mma_ts_k(tmem + kColPR, tmem + kColS, dKQ, kKBlock, 4, idPR, false);
            tc::mma_commit(&bar.mma_pr);
            // Record buffer (i + 1) & 1 held chunk c - 1: its operands were read by the
            // previous update, its vec by the consumers' outputs of chunk c - 1.
            if (i >= 1) {
                if (!wait_or_abort(&bar.o_free, (i - 1) & 1, abort)) { ok = false; break; }
                if (c + 1 < c_end) load_rec(c + 1);
            }
            // The KQ tile is free once [P | R]_c is done.
            if (!wait_or_abort(&bar.mma_pr, i & 1, abort)) { ok = false; break; }
            if (c + 1 < c_end) load_kq(c + 1);
            // [O | S~] (+)= X'_c [Mo; Keff^T]^T, two passes (X_hi, X_lo), N = 192, once X'_c is
            // in tensor memory. A state decayed to exactly zero is overwritten, not rescaled
            // (the O columns were zeroed by the consumers, so they start fresh either way).
            if (!wait_or_abort(&bar.x_ready, i & 1, abort)) { ok = false; break; }
            if (!wait_or_abort(&bar.rec_full[i & 1], (i >> 1) & 1, abort)) { ok = false; break; }
            tc::fence_after_sync();
            const float dC = reinterpret_cast<const float*>(REC(i & 1) + kB2Bytes)[2 * kC];
            const float snext = sigma * dC;
            sigma = decay_renorm(snext) ? 1.f : snext;
            const uint64_t dB2 = tc::desc_kmajor_sw128(smem_u32(REC(i & 1)));
            mma_ts_k(tmem + kColO, tmem + kColXh, dB2, kRBlock, 2, idSO, snext != 0.f);
            mma_ts_k(tmem + kColO, tmem + kColXl, dB2, kRBlock, 2, idSO, true);
            tc::mma_commit(&bar.mma_so);
            if (c + 2 < c_end) load_v(c + 2);   // V_c was read before x_ready
        }
    } else if (warp < 8) {
        // ---------------- consumers
        float sigma = 1.f;      // state = sigma * S~
        OutT* op = reinterpret_cast<OutT*>(p.o);
        for (int c = c_begin; c < c_end; ++c) {
            const int i = c - c_begin;
            const int n = min(kC, T - c * kC);
            const int s = i & 1;
            const float* vec = reinterpret_cast<const float*>(REC(s) + kB2Bytes);
            if (!wait_or_abort(&bar.rec_full[s], (i >> 1) & 1, abort)) { ok = false; break; }
            const float dC = vec[2 * kC];
            const float snext = sigma * dC;
            const bool renorm = decay_renorm(snext);
            const float inv = renorm ? 1.f : 1.f / snext;
            if (!wait_or_abort(&bar.mma_pr, i & 1, abort)) { ok = false; break; }
            tc::fence_after_sync();
            if (!wait_or_abort(&bar.v_full[s], (i >> 1) & 1, abort)) { ok = false; break; }
            // R~_c (kept for this chunk's outputs) and P~_c, both loaded before one wait.
            float rv[32], pv[32];
            tc::tmem_ld32x2(lb + kColPR + kC + 32 * half, lb + kColPR + 32 * half, rv, pv);
            // X'_s = beta_s inv (v_s - sigma d_s P~_s) = a_s v_s - a_s sigma d_s P~_s with
            // a_s = beta_s inv, split into its tf32 high part and the remainder, two tokens per
            // packed fp32 instruction.
            const InT* vt = reinterpret_cast<const InT*>(VT(s)) + row;
            const float2 inv2 = make_float2(inv, inv), sig2 = make_float2(sigma, sigma);
            float xh[32], xl[32];
#pragma unroll
            for (int f = 0; f < 8; ++f) {
                const int t = 32 * half + 4 * f;
                const float4 be = *reinterpret_cast<const float4*>(&vec[kC + t]);
                const float4 dd = *reinterpret_cast<const float4*>(&vec[t]);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int e = 4 * f + 2 * hh;
                    const float2 a2 = __fmul2_rn(hh ? make_float2(be.z, be.w) : make_float2(be.x, be.y), inv2);
                    const float2 bq =
                        __fmul2_rn(__fmul2_rn(a2, sig2), hh ? make_float2(dd.z, dd.w) : make_float2(dd.x, dd.y));
                    const float2 v2 = make_float2(to_f(vt[(t + 2 * hh) * DV]), to_f(vt[(t + 2 * hh + 1) * DV]));
                    const float2 x2 =
                        __ffma2_rn(make_float2(-bq.x, -bq.y), make_float2(pv[e], pv[e + 1]), __fmul2_rn(a2, v2));
                    xh[e] = tc::tf32_hi(x2.x);
                    xh[e + 1] = tc::tf32_hi(x2.y);
                    const float2 l2 = __fadd2_rn(x2, make_float2(-xh[e], -xh[e + 1]));
                    xl[e] = l2.x;
                    xl[e + 1] = l2.y;
                }
            }
            tc::tmem_st16_nowait(lb + kColXh + 32 * half, &xh[0]);
            tc::tmem_st16_nowait(lb + kColXh + 32 * half + 16, &xh[16]);
            tc::tmem_st16_nowait(lb + kColXl + 32 * half, &xl[0]);
            tc::tmem_st16_nowait(lb + kColXl + 32 * half + 16, &xl[16]);
            tc::tmem_st_wait();
            if (renorm && snext != 0.f) {
                // Fold sigma d_C into S~ itself ([P | R]_c has read it); X' = X. A decay of
                // exactly zero is left to the producer, which overwrites S~.
#pragma unroll
                for (int cb = 0; cb < 2; ++cb) {
                    float sv[32];
                    const uint32_t col = lb + kColS + 64 * half + 32 * cb;
                    tc::tmem_ld16(col, *reinterpret_cast<float(*)[16]>(&sv[0]));
                    tc::tmem_ld16(col + 16, *reinterpret_cast<float(*)[16]>(&sv[16]));
#pragma unroll
                    for (int e = 0; e < 32; ++e) sv[e] *= snext;
                    tc::tmem_st32(col, sv);
                }
            }
            tc::fence_before_sync();
            mbar_arrive(&bar.x_ready);
            // Outputs of this chunk once [O | S~]_c is done: o_t = sigma_c d_t R~_t + divO O'_t,
            // tokens 32 half .. +31; the O columns are zeroed again for the next chunk.
            if (!wait_or_abort(&bar.mma_so, i & 1, abort)) { ok = false; break; }
            tc::fence_after_sync();
            float ov[32];
            tc::tmem_ld16(lb + kColO + 32 * half, *reinterpret_cast<float(*)[16]>(&ov[0]));
            tc::tmem_ld16(lb + kColO + 32 * half + 16, *reinterpret_cast<float(*)[16]>(&ov[16]));
            {
                float z[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) z[e] = 0.f;
                tc::tmem_st32(lb + kColO + 32 * half, z);
            }
            const float divO = renorm ? 1.f : snext;
            const float2 div2 = make_float2(divO, divO), sig2o = make_float2(sigma, sigma);
            const size_t tstride = (size_t)p.Hv * DV;   // elements between consecutive tokens
            OutT* orow = op + (((size_t)b * T + (size_t)c * kC + 32 * half) * p.Hv + h) * DV + row;
            const int nt = n - 32 * half;                // tokens of this half inside the prompt
#pragma unroll
            for (int f = 0; f < 8; ++f) {
                const float4 dd = *reinterpret_cast<const float4*>(&vec[32 * half + 4 * f]);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int e = 4 * f + 2 * hh;
                    const float2 rd = __fmul2_rn(sig2o, hh ? make_float2(dd.z, dd.w) : make_float2(dd.x, dd.y));
                    const float2 y = __ffma2_rn(rd, make_float2(rv[e], rv[e + 1]),
                                                __fmul2_rn(div2, make_float2(ov[e], ov[e + 1])));
                    if (e < nt) st_out<OutT>(orow, 0, y.x);
                    orow += tstride;
                    if (e + 1 < nt) st_out<OutT>(orow, 0, y.y);
                    orow += tstride;
                }
            }
            sigma = renorm ? 1.f : snext;
            tc::fence_before_sync();
            mbar_arrive(&bar.o_free);
        }
        if (ok) {
            // Final state = sigma S~ (the last update was waited for above).
            float* dst = p.state_out + (head * DV + row) * DK + 64 * half;
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                float v[32];
                tc::tmem_ld16(lb + kColS + 64 * half + 32 * cb, *reinterpret_cast<float(*)[16]>(&v[0]));
                tc::tmem_ld16(lb + kColS + 64 * half + 32 * cb + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    reinterpret_cast<float4*>(dst + 32 * cb)[q] =
                        make_float4(sigma * v[4 * q], sigma * v[4 * q + 1], sigma * v[4 * q + 2], sigma * v[4 * q + 3]);
            }
        }
    }
    if (!ok) *abort = 1;
    tc::fence_before_sync();
    __syncthreads();
    if (*abort && producer) {
        // Drain: every MMA this thread issued, then the last phase of every copy in flight.
        if (p.status_word) atomicOr(p.status_word, kStatusWaitTimeout);
        tc::mma_commit(&bar.drain);
        mbar_wait_bounded(&bar.drain, 0, kMaxPolls);
        if (n_kq) mbar_wait_bounded(&bar.kq_full, (n_kq - 1) & 1, kMaxPolls);
        if (n_rec0) mbar_wait_bounded(&bar.rec_full[0], (n_rec0 - 1) & 1, kMaxPolls);
        if (n_rec1) mbar_wait_bounded(&bar.rec_full[1], (n_rec1 - 1) & 1, kMaxPolls);
        if (n_v0) mbar_wait_bounded(&bar.v_full[0], (n_v0 - 1) & 1, kMaxPolls);
        if (n_v1) mbar_wait_bounded(&bar.v_full[1], (n_v1 - 1) & 1, kMaxPolls);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// Workspace pointers: KQ tiles first, then the records.
inline float* ws_kq_of(const VerifyArgs&, void* ws) { return static_cast<float*>(ws); }
inline unsigned char* ws_rec_of(const VerifyArgs& a, void* ws) {
    return static_cast<unsigned char*>(ws) + (size_t)a.B * a.Hk * n_chunks_of(a.T) * kKQBytes;
}

// Chunks [c0, c1) of every (sequence, key head).
template <typename InT>
cudaError_t launch_prep(const VerifyArgs& a, void* workspace, int c0, int c1, cudaStream_t stream) {
    cudaError_t e = ensure_smem_attr<gdn_prefill_prep_kernel<InT>>((int)sizeof(PrepSmem));
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(c1 - c0), a.Hk, a.B);
    gdn_prefill_prep_kernel<InT><<<grid, kPrepThreads, sizeof(PrepSmem), stream>>>(a, ws_kq_of(a, workspace),
                                                                                    ws_rec_of(a, workspace), c0);
    return cudaGetLastError();
}

// Chunks [c0, c1), from the state in a.state_in (zero when NULL) to a.state_out.
template <typename InT, typename OutT>
cudaError_t launch_scan(const VerifyArgs& a, void* workspace, int c0, int c1, cudaStream_t stream) {
    cudaError_t e = ensure_smem_attr<gdn_prefill_scan_kernel<InT, OutT>>((int)scan_smem_bytes<InT>());
    if (e != cudaSuccess) return e;
    CUtensorMap v_map;
    e = tc::encode_tmap_tokens(&v_map, a.v, sizeof(InT) == 2, DV, a.Hv, a.T, a.B, kC);
    if (e != cudaSuccess) return e;
    dim3 grid(a.Hv, a.B);
    gdn_prefill_scan_kernel<InT, OutT><<<grid, kScanThreads, scan_smem_bytes<InT>(), stream>>>(
        v_map, a, ws_kq_of(a, workspace), ws_rec_of(a, workspace), c0, c1);
    return cudaGetLastError();
}

cudaError_t prepare_range(const VerifyArgs& a, void* workspace, int c0, int c1, cudaStream_t stream) {
    return a.in_bf16 ? launch_prep<__nv_bfloat16>(a, workspace, c0, c1, stream)
                     : launch_prep<float>(a, workspace, c0, c1, stream);
}

cudaError_t scan_range(const VerifyArgs& a, void* workspace, int c0, int c1, cudaStream_t stream) {
    if (a.in_bf16)
        return a.out_bf16 ? launch_scan<__nv_bfloat16, __nv_bfloat16>(a, workspace, c0, c1, stream)
                          : launch_scan<__nv_bfloat16, float>(a, workspace, c0, c1, stream);
    return a.out_bf16 ? launch_scan<float, __nv_bfloat16>(a, workspace, c0, c1, stream)
                      : launch_scan<float, float>(a, workspace, c0, c1, stream);
}

// The prompt is split into pieces of whole chunks: the scan of piece i (one CTA and a whole SM
// per value head) runs on a stream of the greatest priority while the preparation of piece i + 1
// runs on the caller's stream. Each time the GPU drains at the end of a preparation, the
// scan's CTAs are dispatched first and the next preparation fills the SMs the scan leaves (a
// preparation CTA does not fit beside a scan CTA's shared memory). No kernel waits on another:
// events order the pieces, so the worst case is the two phases one after the other.
constexpr int kMaxPieces = 4;        // measured on the 32768-token prompt: 4 pieces 2.07 ms,
                                     // 8 pieces 2.11, 16 pieces 2.25, one piece 2.65
constexpr int kPieceMinChunks = 32;

struct PieceStreams {
    cudaStream_t hi = nullptr;
    cudaEvent_t ev[kMaxPieces + 1] = {};
};

// The stream and events of the current device, created on first use and kept for the life of
// the process. The caller holds launch_prefill's mutex, which guards them.
cudaError_t piece_streams(PieceStreams** out) {
    constexpr int kMaxDevices = 64;
    static PieceStreams ps[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    PieceStreams& p = ps[dev];
    if (!p.hi) {
        int least = 0, greatest = 0;
        e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
        if (e != cudaSuccess) return e;
        for (int i = 0; i <= kMaxPieces; ++i) {
            if (p.ev[i]) continue;
            e = cudaEventCreateWithFlags(&p.ev[i], cudaEventDisableTiming);
            if (e != cudaSuccess) return e;
        }
        e = cudaStreamCreateWithPriority(&p.hi, cudaStreamNonBlocking, greatest);
        if (e != cudaSuccess) return e;
    }
    *out = &p;
    return cudaSuccess;
}

// Fixed scratch for gdn_chunk_prefill_noalloc. It is a module-scope device array, so every
// GPU that loads this library holds it (kNoAllocScratchBytes) until the process exits, and
// every call of that entry point on one GPU reuses the same bytes.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device. In host code the array's name
// is only a host-side stand-in, so the address is asked of the runtime, once per device (with
// that device current), and cached.
cudaError_t noalloc_scratch_address(void** out) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_prefill_noalloc(const VerifyArgs& a, int chunk, cudaStream_t stream) {
    // Nothing in the scratch has to start at zero: the prep kernel writes every workspace
    // element the scan kernel reads, on the same stream, before the scan reads it.
    void* ws = nullptr;
    cudaError_t e = noalloc_scratch_address(&ws);
    if (e != cudaSuccess) return e;
    return launch_prefill(a, chunk, ws, kNoAllocScratchBytes, stream);
}

int check_prefill_shape(const gdn_shape* s, int chunk) {
    if (!s) return -1;
    if (chunk != kC) return -1;
    if (s->d_k != DK || s->d_v != DV) return -1;
    return 0;
}

size_t prefill_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv, int chunk) {
    (void)dk;
    (void)dv;
    (void)chunk;
    const size_t nch = n_chunks_of(T);
    return (size_t)B * Hk * nch * kKQBytes + (size_t)B * Hv * nch * kRecBytes;
}

int prefill_pieces(long long T) {
    if (T <= 0) return 0;
    const long long nch = ((long long)T + kC - 1) / kC;
    return (int)std::max(1LL, std::min((long long)kMaxPieces, nch / kPieceMinChunks));
}

cudaError_t launch_prefill_prepare(const VerifyArgs& a, void* workspace, cudaStream_t stream) {
    return prepare_range(a, workspace, 0, (int)n_chunks_of(a.T), stream);
}

cudaError_t launch_prefill_scan(const VerifyArgs& a, void* workspace, cudaStream_t stream) {
    return scan_range(a, workspace, 0, (int)n_chunks_of(a.T), stream);
}

cudaError_t launch_prefill(const VerifyArgs& a, int chunk, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
    (void)chunk;
    (void)workspace_bytes;
    const int nch = (int)n_chunks_of(a.T);
    const int np = prefill_pieces(a.T);
    if (np == 1) {
        cudaError_t e = launch_prefill_prepare(a, workspace, stream);
        return e == cudaSuccess ? launch_prefill_scan(a, workspace, stream) : e;
    }
    auto bound = [&](int i) { return (int)((long long)nch * i / np); };
    // Under stream capture the pieces run in order on the caller's stream, with the same
    // bounds (so the same bits as an eager call). The side stream is shared by every caller on
    // the device: joined to a capture, it would stay part of it until the capture ends, and an
    // eager call from another thread in that window would queue into the capture.
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return e;
    if (cap != cudaStreamCaptureStatusNone) {
        VerifyArgs ai = a;
        for (int i = 0; i < np && e == cudaSuccess; ++i) {
            if (i > 0) ai.state_in = a.state_out;
            e = prepare_range(a, workspace, bound(i), bound(i + 1), stream);
            if (e == cudaSuccess) e = scan_range(ai, workspace, bound(i), bound(i + 1), stream);
        }
        return e;
    }
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    PieceStreams* ps = nullptr;
    e = piece_streams(&ps);
    if (e != cudaSuccess) return e;
    // Piece 0's preparation on the caller's stream, after the caller's earlier work.
    e = prepare_range(a, workspace, 0, bound(1), stream);
    if (e == cudaSuccess) e = cudaEventRecord(ps->ev[0], stream);
    VerifyArgs ai = a;
    for (int i = 0; i < np && e == cudaSuccess; ++i) {
        e = cudaStreamWaitEvent(ps->hi, ps->ev[i], 0);
        if (e != cudaSuccess) break;
        // Piece i starts from the state piece i - 1 left in state_out.
        if (i > 0) ai.state_in = a.state_out;
        e = scan_range(ai, workspace, bound(i), bound(i + 1), ps->hi);
        if (e != cudaSuccess || i + 1 == np) break;
        e = prepare_range(a, workspace, bound(i + 1), bound(i + 2), stream);
        if (e == cudaSuccess) e = cudaEventRecord(ps->ev[i + 1], stream);
    }
    // The caller's stream resumes after the last scan, also when a launch failed on the way
    // (the work already queued on the side stream then still precedes the caller's next work).
    cudaError_t j = cudaEventRecord(ps->ev[np], ps->hi);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(stream, ps->ev[np], 0);
    return e != cudaSuccess ? e : j;
}

}  // namespace gdn
