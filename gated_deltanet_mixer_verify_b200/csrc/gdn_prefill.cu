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
// Two kernels:
//   gdn_prefill_prep_kernel, one CTA per (sequence, value head, chunk), all in parallel: the
//     state-independent part. Normalised keys / queries and their Gram matrix (tensor cores);
//     then Mo and Keff^T without forming Tm: both solve x (I + A) = y for a row vector y (a row
//     of Cq, or the column exp(G_C - G_t) khat_t[j] for one key dimension j), which one thread
//     does by right-looking back substitution in registers. The results go to the workspace in
//     the exact shared-memory image the scan consumes (one bulk store each).
//   gdn_prefill_scan_kernel, one CTA per (sequence, value head), chunk after chunk, warp
//     specialised: warp 8 streams the chunk operands in (bulk copies and a TMA tensor copy of
//     V) and issues the tensor-core MMAs; warps 0-7 form X and write the outputs. The state
//     lives in tensor memory (fp32) as the A operand of P | R and the accumulator of the
//     update. Its per-chunk decay d_C is carried in a scalar sigma (state = sigma * S~) and
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
//         rows 0..127 Keff^T (row j = Keff_s[j] over s), rows 128..191 Mo (row t = Mo[t][s]);
//         values rounded to the nearest tf32.
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

struct __align__(1024) PrepSmem {
    float KQ[2 * kC * DK];     // [khat; qhat] SW128 image; afterwards the staging of B2
    float A[kC][kApad];        // strictly lower A
    float G[kC], Beta[kC], Ec[kC];
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

template <typename InT>
__global__ void __launch_bounds__(kPrepThreads, 2)
    gdn_prefill_prep_kernel(const VerifyArgs p, float* __restrict__ ws_kq, unsigned char* __restrict__ ws_rec) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    PrepSmem& sm = *reinterpret_cast<PrepSmem*>(smem_raw);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int c = blockIdx.x;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int T = p.T;
    const int grp = p.Hv / p.Hk;
    const int g = h / grp;
    const size_t nch = n_chunks_of(T);
    const int t0 = c * kC;
    const int n = min(kC, T - t0);   // tokens in this chunk
    const size_t unit = ((size_t)b * p.Hv + h) * nch + c;
    const bool store_kq = (h % grp) == 0;   // one value head per key head writes the KQ tile

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

    // 1. Gates of this chunk (warps 0, 1: token t = tid), loads issued first.
    float gl = 0.f, be = 0.f;
    if (warp < 2 && tid < n) {
        const size_t gi = ((size_t)b * T + t0 + tid) * p.Hv + h;
        gl = -expf(p.A_log[h]) * softplus_f(ld_in<InT>(p.a, gi) + p.dt_bias[h]);
        be = 1.f / (1.f + expf(-ld_in<InT>(p.b, gi)));
    }
    // khat / qhat rows: 16 threads x 8 columns per row, 16 rows per pass, all loads in flight.
    {
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
            *reinterpret_cast<float4*>(&sm.KQ[tc::sw128_offset(r, 8 * c16, 2 * kC) / 4]) =
                make_float4(x[it][0] * inv, x[it][1] * inv, x[it][2] * inv, x[it][3] * inv);
            *reinterpret_cast<float4*>(&sm.KQ[tc::sw128_offset(r, 8 * c16 + 4, 2 * kC) / 4]) =
                make_float4(x[it][4] * inv, x[it][5] * inv, x[it][6] * inv, x[it][7] * inv);
        }
    }
    if (warp < 2) {
        float Gs = gl;   // inclusive prefix sum within the warp; warp 1 adds warp 0's total below
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(kFull, Gs, off);
            if (lane >= off) Gs += y;
        }
        sm.G[tid] = Gs;
        sm.Beta[tid] = be;
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem;

    // 2. Gram on the tensor cores: D (128 x 64) = [Khat; Qhat] Khat^T, one tf32 pass; the KQ
    // tile goes to the workspace at the same time.
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
    if (tid == 32 && store_kq) {
        bulk_s2g(ws_kq + (((size_t)b * p.Hk + g) * nch + c) * (kKQBytes / 4), sm.KQ, kKQBytes);
        bulk_commit();
    }
    if (warp == 1) sm.G[tid] += sm.G[31];
    __syncthreads();
    if (tid < kC) {
        const float GC = sm.G[n - 1];
        sm.Ec[tid] = tid < n ? expf(GC - sm.G[tid]) : 0.f;
        float* vec = reinterpret_cast<float*>(ws_rec + unit * kRecBytes + kB2Bytes);
        vec[tid] = tid < n ? expf(sm.G[tid]) : 0.f;
        vec[kC + tid] = sm.Beta[tid];
        if (tid == 0) vec[2 * kC] = expf(GC);
    }
    __syncthreads();

    // 3. Right-hand sides. Warps 0, 1: Gram rows t -> A row t in shared memory. Warps 2, 3:
    // Gram rows 64 + t -> Cq row t (registers). Warps 4-7: key dimension j -> exp(G_C - G_s)
    // khat_s[j] (registers).
    bool ok = mbar_wait_bounded(&sm.mma_done, 0, kMaxPolls);
    tc::fence_after_sync();
    float2 acc[kC / 2];
    if (warp < 4) {
        float gv[kC];
#pragma unroll
        for (int cb = 0; cb < kC; cb += 16)
            tc::tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + cb, *reinterpret_cast<float(*)[16]>(&gv[cb]));
        const int t = (32 * warp + lane) & (kC - 1);
        const float Gt = sm.G[t];
        if (warp < 2) {
            const float bt = sm.Beta[t];
#pragma unroll
            for (int s4 = 0; s4 < kC; s4 += 4) {
                float a[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int s = s4 + e;
                    a[e] = (s < t && t < n) ? bt * expf(Gt - sm.G[s]) * gv[s] : 0.f;
                }
                *reinterpret_cast<float4*>(&sm.A[t][s4]) = make_float4(a[0], a[1], a[2], a[3]);
            }
        } else {
#pragma unroll
            for (int s2 = 0; s2 < kC / 2; ++s2) {
                const int s = 2 * s2;
                acc[s2].x = (s <= t && t < n) ? expf(Gt - sm.G[s]) * gv[s] : 0.f;
                acc[s2].y = (s + 1 <= t && t < n) ? expf(Gt - sm.G[s + 1]) * gv[s + 1] : 0.f;
            }
        }
    } else {
        const int j = tid - 128;
#pragma unroll
        for (int s2 = 0; s2 < kC / 2; ++s2) {
            const int s = 2 * s2;
            acc[s2].x = sm.Ec[s] * sm.KQ[tc::sw128_offset(s, j, 2 * kC) / 4];
            acc[s2].y = sm.Ec[s + 1] * sm.KQ[tc::sw128_offset(s + 1, j, 2 * kC) / 4];
        }
    }
    if (tid == 32 && store_kq) bulk_wait_read_all();   // the KQ store has read the tile
    tc::fence_before_sync();
    __syncthreads();

    // 4. Solves: warps 2, 3 give Mo rows, warps 4-7 Keff^T rows; staged (rounded to tf32) over
    // the KQ tile, which is no longer read, in the record's B2 image.
    if (ok && warp >= 2) {
        solve_unit_lower_row(acc, sm.A);
        const int row = warp < 4 ? DK + (tid - 64) : tid - 128;
#pragma unroll
        for (int f = 0; f < kC / 4; ++f) {
            const float4 v = make_float4(tc::tf32_rna(acc[2 * f].x), tc::tf32_rna(acc[2 * f].y),
                                         tc::tf32_rna(acc[2 * f + 1].x), tc::tf32_rna(acc[2 * f + 1].y));
            *reinterpret_cast<float4*>(&sm.KQ[tc::sw128_offset(row, 4 * f, kRecRows) / 4]) = v;
        }
    }
    tc::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
        if (ok) {
            bulk_s2g(ws_rec + unit * kRecBytes, sm.KQ, kB2Bytes);
            bulk_commit();
            bulk_wait_all();
        } else if (p.status_word) {
            atomicOr(p.status_word, kStatusWaitTimeout);
        }
    }
    if (tid == 32 && store_kq) bulk_wait_all();
    tc::fence_before_sync();
    __syncthreads();
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
    uint64_t mma_p, mma_r, mma_s, mma_o, drain;
    uint64_t x_ready, o_free;           // 256 arrivals each
    uint32_t tmem;
    int abort;
};
static_assert(kOffBar + sizeof(ScanBars) <= kOffRec1, "barriers overflow the record slack");

// TMEM columns: S~ 0..127, P 128..191, R (two buffers) 192..319, O 320..383, X_hi 384..447,
// X_lo 448..511.
constexpr uint32_t kColS = 0, kColP = 128, kColR = 192, kColO = 320, kColXh = 384, kColXl = 448;
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

// Outputs of chunk c for state row `row`, tokens 32 half .. +31 (those below n):
// o_t = rd_t R~_t + divO O'_t, with R~ in tensor-memory buffer c % 2 and O' in the O columns.
template <typename OutT>
__device__ __forceinline__ void scan_outputs(const VerifyArgs& p, uint32_t lb, int b, int h, int half, int row, int c,
                                             int n, const float (&rd)[32], float divO) {
    OutT* op = reinterpret_cast<OutT*>(p.o);
    const size_t base = ((size_t)b * p.T + (size_t)c * kC + 32 * half) * p.Hv + h;
    const uint32_t rcol = kColR + (uint32_t)(c & 1) * kC + 32 * half;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        float rv[16], ov[16];
        tc::tmem_ld16(lb + rcol + 16 * q, rv);
        tc::tmem_ld16(lb + kColO + 32 * half + 16 * q, ov);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int u = 16 * q + e;
            if (32 * half + u < n)
                st_out<OutT>(op, (base + (size_t)u * p.Hv) * DV + row, fmaf(rd[u], rv[e], divO * ov[e]));
        }
    }
}

template <typename InT, typename OutT>
__global__ void __launch_bounds__(kScanThreads, 1)
    gdn_prefill_scan_kernel(const __grid_constant__ CUtensorMap v_map, const VerifyArgs p,
                            const float* __restrict__ ws_kq, const unsigned char* __restrict__ ws_rec) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    constexpr uint32_t kVBytes = v_tile_bytes<InT>();
    ScanBars& bar = *reinterpret_cast<ScanBars*>(smem_raw + kOffBar);
    float* KQ = reinterpret_cast<float*>(smem_raw + kOffKQ);
    // Record buffer i at smem_raw + kOffRec0 + i * kRecStride, V buffer i at kOffV0 + i * kVBytes.
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
        mbar_init(&bar.mma_p, 1);
        mbar_init(&bar.mma_r, 1);
        mbar_init(&bar.mma_s, 1);
        mbar_init(&bar.mma_o, 1);
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
    auto load_rec = [&](int c) {
        const int s = c & 1;
        mbar_arrive_expect_tx(&bar.rec_full[s], kRecBytes);
        bulk_g2s(REC(s), rec_src + (size_t)c * kRecBytes, kRecBytes, &bar.rec_full[s]);
        if (s) ++n_rec1; else ++n_rec0;
    };
    auto load_v = [&](int c) {
        const int s = c & 1;
        mbar_arrive_expect_tx(&bar.v_full[s], kVBytes);
        tc::tma_load_4d(VT(s), &v_map, 0, h, c * kC, b, &bar.v_full[s]);
        if (s) ++n_v1; else ++n_v0;
    };
    if (producer) {
        load_kq(0);
        load_rec(0);
        load_v(0);
        if (nch > 1) {
            load_rec(1);
            load_v(1);
        }
    }

    // Consumer geometry: warp w owns TMEM lanes 32 (w % 4) .. +31 (state rows) and token
    // columns 32 (w / 4) .. +31 of each chunk.
    const int q4 = warp & 3;
    const int half = (warp >> 2) & 1;
    const int row = 32 * q4 + lane;
    const uint32_t lb = tmem + ((uint32_t)(32 * q4) << 16);

    // Initial state (zero when state_in is NULL) into tensor memory, columns 64 half .. +63.
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
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();

    bool ok = true;
    if (producer) {
        // ---------------- producer / MMA issuer
        const uint32_t idPR = tc::idesc_tf32(DV, kC), idS = tc::idesc_tf32(DV, DK), idO = tc::idesc_tf32(DV, kC);
        const uint64_t dKQ = tc::desc_kmajor_sw128(smem_u32(KQ));
        auto issue_o = [&](int c) {   // O_c = X'_c Mo_c^T, two passes
            const uint64_t dMo = tc::desc_kmajor_sw128(smem_u32(REC(c & 1)) + DK * 128);
            mma_ts_k(tmem + kColO, tmem + kColXh, dMo, kRBlock, 2, idO, false);
            mma_ts_k(tmem + kColO, tmem + kColXl, dMo, kRBlock, 2, idO, true);
            tc::mma_commit(&bar.mma_o);
        };
        for (int c = 0; c < nch && ok; ++c) {
            if (!wait_or_abort(&bar.kq_full, c & 1, abort)) { ok = false; break; }
            tc::fence_after_sync();
            // P_c = S~ Khat^T, then R_c = S~ Qhat^T (A = S~ in tensor memory, one pass).
            mma_ts_k(tmem + kColP, tmem + kColS, dKQ, kKBlock, 4, idPR, false);
            tc::mma_commit(&bar.mma_p);
            // R_c and O_{c-1} overwrite what the outputs of chunk c-2 read, and the record
            // buffer refilled below held the vec the consumers copied in chunk c-1.
            if (c >= 1 && !wait_or_abort(&bar.o_free, (c - 1) & 1, abort)) { ok = false; break; }
            mma_ts_k(tmem + kColR + (uint32_t)(c & 1) * kC, tmem + kColS, dKQ + ((kC * 128) >> 4), kKBlock, 4, idPR,
                     false);
            tc::mma_commit(&bar.mma_r);
            if (c >= 1) issue_o(c - 1);
            // The KQ tile is free once R_c is done.
            if (!wait_or_abort(&bar.mma_r, c & 1, abort)) { ok = false; break; }
            if (c + 1 < nch) load_kq(c + 1);
            // Record buffer (c + 1) & 1 is free once O_{c-1} is done.
            if (c >= 1) {
                if (!wait_or_abort(&bar.mma_o, (c - 1) & 1, abort)) { ok = false; break; }
                if (c + 1 < nch) load_rec(c + 1);
            }
            // S~ += X'_c Keff_c, two passes, once X'_c is in tensor memory.
            if (!wait_or_abort(&bar.x_ready, c & 1, abort)) { ok = false; break; }
            if (!wait_or_abort(&bar.rec_full[c & 1], (c >> 1) & 1, abort)) { ok = false; break; }
            tc::fence_after_sync();
            {
                const uint64_t dKe = tc::desc_kmajor_sw128(smem_u32(REC(c & 1)));
                mma_ts_k(tmem + kColS, tmem + kColXh, dKe, kRBlock, 2, idS, true);
                mma_ts_k(tmem + kColS, tmem + kColXl, dKe, kRBlock, 2, idS, true);
                tc::mma_commit(&bar.mma_s);
            }
            if (c + 2 < nch) load_v(c + 2);   // V_c was read before x_ready
            if (!wait_or_abort(&bar.mma_s, c & 1, abort)) { ok = false; break; }
        }
        if (ok) {
            if (wait_or_abort(&bar.o_free, (nch - 1) & 1, abort)) issue_o(nch - 1);
            else ok = false;
        }
    } else if (warp < 8) {
        // ---------------- consumers
        float sigma = 1.f;      // state = sigma * S~
        float rd[32];           // sigma_c d_t for the previous chunk's outputs
        float divO = 1.f;       // O = divO * (X' Mo^T) for the previous chunk
        int n_prev = 0;
#pragma unroll
        for (int e = 0; e < 32; ++e) rd[e] = 0.f;
        for (int c = 0; c < nch; ++c) {
            const int t0 = c * kC;
            const int n = min(kC, T - t0);
            const int s = c & 1;
            const float* vec = reinterpret_cast<const float*>(REC(s) + kB2Bytes);
            if (!wait_or_abort(&bar.rec_full[s], (c >> 1) & 1, abort)) { ok = false; break; }
            const float dC = vec[2 * kC];
            const float snext = sigma * dC;
            const bool renorm = !(snext >= kRenormBelow);
            const float inv = renorm ? 1.f : 1.f / snext;
            if (!wait_or_abort(&bar.mma_p, c & 1, abort)) { ok = false; break; }
            tc::fence_after_sync();
            if (!wait_or_abort(&bar.v_full[s], (c >> 1) & 1, abort)) { ok = false; break; }
            const InT* vt = reinterpret_cast<const InT*>(VT(s)) + row;
            // X'_s = beta_s inv (v_s - sigma d_s P~_s), split into tf32 high part and remainder.
            float xh[32], xl[32];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float pv[16];
                tc::tmem_ld16(lb + kColP + 32 * half + 16 * q, pv);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int t = 32 * half + 16 * q + e;
                    const float x = vec[kC + t] * inv * fmaf(-vec[t] * sigma, pv[e], to_f(vt[t * DV]));
                    xh[16 * q + e] = tc::tf32_hi(x);
                    xl[16 * q + e] = x - xh[16 * q + e];
                }
            }
            // X_{c-1} must have been read by O_{c-1} before it is overwritten.
            if (c >= 1) {
                if (!wait_or_abort(&bar.mma_o, (c - 1) & 1, abort)) { ok = false; break; }
                tc::fence_after_sync();
            }
            if (renorm) {
                // Fold sigma d_C into S~ itself (R_c must have read S~ first); X' = X.
                if (!wait_or_abort(&bar.mma_r, c & 1, abort)) { ok = false; break; }
                tc::fence_after_sync();
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
            tc::tmem_st32(lb + kColXh + 32 * half, xh);
            tc::tmem_st32(lb + kColXl + 32 * half, xl);
            tc::fence_before_sync();
            mbar_arrive(&bar.x_ready);
            if (c >= 1) scan_outputs<OutT>(p, lb, b, h, half, row, c - 1, n_prev, rd, divO);
#pragma unroll
            for (int e = 0; e < 32; ++e) rd[e] = sigma * vec[32 * half + e];
            divO = renorm ? 1.f : snext;
            sigma = renorm ? 1.f : snext;
            n_prev = n;
            tc::fence_before_sync();
            mbar_arrive(&bar.o_free);
        }
        if (ok && wait_or_abort(&bar.mma_o, (nch - 1) & 1, abort)) {
            tc::fence_after_sync();
            scan_outputs<OutT>(p, lb, b, h, half, row, nch - 1, n_prev, rd, divO);
            // Final state = sigma S~.
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
        } else {
            ok = false;
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

template <typename InT, typename OutT>
cudaError_t launch_tc_prefill(const VerifyArgs& a, void* workspace, cudaStream_t stream) {
    const size_t nch = n_chunks_of(a.T);
    float* ws_kq = static_cast<float*>(workspace);
    unsigned char* ws_rec = static_cast<unsigned char*>(workspace) + (size_t)a.B * a.Hk * nch * kKQBytes;
    // Per call: the attribute belongs to the function on the current device.
    cudaError_t e = cudaFuncSetAttribute(gdn_prefill_prep_kernel<InT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(PrepSmem));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gdn_prefill_scan_kernel<InT, OutT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)scan_smem_bytes<InT>());
    if (e != cudaSuccess) return e;
    CUtensorMap v_map;
    e = tc::encode_tmap_tokens(&v_map, a.v, sizeof(InT) == 2, DV, a.Hv, a.T, a.B, kC);
    if (e != cudaSuccess) return e;
    dim3 pgrid((unsigned)nch, a.Hv, a.B);
    gdn_prefill_prep_kernel<InT><<<pgrid, kPrepThreads, sizeof(PrepSmem), stream>>>(a, ws_kq, ws_rec);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 sgrid(a.Hv, a.B);
    gdn_prefill_scan_kernel<InT, OutT><<<sgrid, kScanThreads, scan_smem_bytes<InT>(), stream>>>(v_map, a, ws_kq,
                                                                                                  ws_rec);
    return cudaGetLastError();
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

cudaError_t launch_prefill(const VerifyArgs& a, int chunk, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
    (void)chunk;
    (void)workspace_bytes;
    if (a.in_bf16)
        return a.out_bf16 ? launch_tc_prefill<__nv_bfloat16, __nv_bfloat16>(a, workspace, stream)
                          : launch_tc_prefill<__nv_bfloat16, float>(a, workspace, stream);
    return a.out_bf16 ? launch_tc_prefill<float, __nv_bfloat16>(a, workspace, stream)
                      : launch_tc_prefill<float, float>(a, workspace, stream);
}

}  // namespace gdn
