// gdn_verify_tc.cu -- tensor-core form of the verify mixer for d_k = d_v = 128, T <= 8.
//
// Same block-form math as gdn_verify.cu (dots against the block's initial state, a T x T
// unit-triangular solve, folded commit keys). The 2T dots per state row are a dense
// contraction, P = S_0 [Khat; Qhat]^T (128 x 128 times 128 x 2T), so they run on the 5th-
// generation tensor cores (tcgen05.mma, kind::tf32, fp32 accumulator in tensor memory) in
// three passes, S_hi B_hi + S_hi B_lo + S_lo B_hi, where x_hi is x with its low 13 mantissa
// bits cleared and x_lo = x - x_hi: this keeps the products accurate to about 2^-20 of fp32
// (a single tf32 pass would be ~2^-11). The CUDA cores only split the state, run the small
// per-head algebra, form outputs and write the committed rows.
//
// Shared memory holds the raw fp32 state tile (TMA, 128-byte swizzle): a kind::tf32 MMA
// reads a 32-bit container as its truncated tf32 value, so that tile serves directly as S_hi.
// S_lo = S - S_hi is formed by the threads and stored in tensor memory, where the third pass
// takes its A operand. That keeps a CTA at ~100 KB of shared memory and 256 tensor-memory
// columns, so two CTAs (16 warps) share an SM and overlap one head's copies and algebra with
// the other's MMAs and commit. One CTA per (sequence, head); each CTA also prefetches into L2
// the inputs of the CTA one resident wave ahead, and splits its state as soon as it lands,
// while warp 0 is still on the gate chain.
// Every mbarrier wait is bounded; a timeout sets GDN_STATUS_WAIT_TIMEOUT, suppresses the
// CTA's global writes, drains its copy and MMAs (bounded) and frees its tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {
using namespace dev;

constexpr int kThreads = 256;
constexpr int DK = 128;
constexpr int DV = 128;
constexpr int TM = 8;                  // block length bound (N = 2 TM = 16)
constexpr int NB = 2 * TM;             // rows of the B operand: khat_0..7, qhat_0..7
constexpr uint32_t kTileBytes = DV * DK * 4;
constexpr uint32_t kMaxPolls = 1u << 24;

struct __align__(1024) TcSmem {
    float S[DV * DK];        // raw fp32 state tile, SW128 K-major (4 blocks of [128 rows][32])
    float B2[2 * NB * DK];   // rows 0..15: [khat; qhat] high parts, rows 16..31: low parts;
                             // SW128 K-major (4 blocks of [32 rows][32])
    float KQ[NB][DK];        // khat, qhat in plain fp32 (Gram, Keff, stash)
    float Keff[TM][DK];
    float2 X2[DV][TM];       // (x_s, x_s) per state row: ready-made operands of the packed FMAs
    // Commit-on-next-verify: the previous block's stash for this head as stored (khat'_t rows,
    // scaled in place to KP_t = c_t khat'_t; the decays G'; the u'_t rows), and W = KP [khat;
    // qhat]^T, the correction of the dots for the committed state. With the gated norm instead
    // (never both), PS holds the block's gate rows z_t (input dtype) and then the d_v weights.
    float PS[2 * TM * DK + TM];
    float W[TM][NB];
    float NSS[8][TM / 2];    // gated norm: per warp, its 4 tokens' partial sums of squares
    float Gram[NB][TM];
    float G[TM], Beta[TM], D[TM];
    float A[TM][TM], Cq[TM][TM], Tm[TM][TM], Mo[TM][TM], E[TM][TM];
    float Ec[TM];            // decay from token t to the last accepted token
    float DL;
    float PD;                // decay of the previous block at its accept count L'
    int L;
    int PL;                  // L' (0 for an out-of-range count)
    int fail;                // the state copy's bounded wait ran out
    int pfail;               // the previous stash copy's bounded wait ran out
    uint32_t tmem;           // 256 columns: S_lo (A operand of the third pass) at 0..127, the
                             // dots (128 lanes x 32) at 128..159
    uint64_t full;
    uint64_t mma_done;
    uint64_t prev_full;      // the previous stash has landed in PS
};

__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Arrive at named barrier `id` (expecting nthreads) without waiting for it.
__device__ __forceinline__ void named_arrive(int id, int nthreads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Committed rows for a compile-time number LL of accepted tokens: S_L = d S_0 + sum_{s<LL}
// x_s Keff_s (LL = 0: S_0 unchanged). One warp per 16 rows, a lane per 16-byte column chunk.
// PRE: S_0 is first replaced by the previous block committed at its count L' = Lp,
// S' = pd S_0 + sum_{t<Lp} u'_t KP_t^T (stash rows in PS, u' rows from offset off_u).
template <int LL, bool PRE>
__device__ __forceinline__ void commit_rows(const TcSmem& sm, float* dst, int warp, int lane, float dl, int Lp,
                                            float pd, int off_u) {
    const int chunk = lane;   // columns 4*chunk .. +3
    const int kb = chunk >> 3, c = chunk & 7;
    float4 ke[LL > 0 ? LL : 1];
#pragma unroll
    for (int s = 0; s < LL; ++s) ke[s] = *reinterpret_cast<const float4*>(&sm.Keff[s][4 * chunk]);
    float4 kp[PRE ? TM : 1];
    if (PRE) {
#pragma unroll
        for (int t = 0; t < TM; ++t)
            kp[t] = (t < Lp) ? *reinterpret_cast<const float4*>(&sm.PS[t * DK + 4 * chunk]) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float2 dl2 = make_float2(dl, dl);
#pragma unroll 4
    for (int i = 0; i < DV / 8; ++i) {
        const int row = warp + 8 * i;
        const float4 sv =
            *reinterpret_cast<const float4*>(&sm.S[(kb * DV * 128 + row * 128 + ((c ^ (row & 7)) << 4)) / 4]);
        float2 r0 = make_float2(sv.x, sv.y), r1 = make_float2(sv.z, sv.w);
        if (PRE) {
            const float2 pd2 = make_float2(pd, pd);
            r0 = __fmul2_rn(r0, pd2);
            r1 = __fmul2_rn(r1, pd2);
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                if (t < Lp) {
                    const float u = sm.PS[off_u + t * DV + row];   // the same word for the whole warp
                    const float2 u2 = make_float2(u, u);
                    r0 = __ffma2_rn(u2, make_float2(kp[t].x, kp[t].y), r0);
                    r1 = __ffma2_rn(u2, make_float2(kp[t].z, kp[t].w), r1);
                }
            }
        }
        if (LL > 0) {
            r0 = __fmul2_rn(r0, dl2);
            r1 = __fmul2_rn(r1, dl2);
#pragma unroll
            for (int s = 0; s < LL; s += 2) {
                const float4 xp = *reinterpret_cast<const float4*>(&sm.X2[row][s]);
                const float2 xa = make_float2(xp.x, xp.y);
                r0 = __ffma2_rn(xa, make_float2(ke[s].x, ke[s].y), r0);
                r1 = __ffma2_rn(xa, make_float2(ke[s].z, ke[s].w), r1);
                if (s + 1 < LL) {
                    const float2 xb = make_float2(xp.z, xp.w);
                    r0 = __ffma2_rn(xb, make_float2(ke[s + 1].x, ke[s + 1].y), r0);
                    r1 = __ffma2_rn(xb, make_float2(ke[s + 1].z, ke[s + 1].w), r1);
                }
            }
        }
        __stcs(reinterpret_cast<float4*>(dst + (size_t)row * DK) + chunk, make_float4(r0.x, r0.y, r1.x, r1.y));
    }
}

// Gated norm: nw silu(z_t) for this thread's row and its 4 tokens, from the gate rows and
// weights staged in PS (waits for their copies, bounded; a timeout sets pfail).
template <typename InT>
__device__ __forceinline__ void gate_factors(TcSmem& sm, const VerifyArgs& p, int T, int tid, float (&gz)[TM / 2]) {
    if (!mbar_wait_bounded(&sm.prev_full, 0, kMaxPolls)) sm.pfail = 1;
    const int row = tid & (DV - 1);
    const InT* zs = reinterpret_cast<const InT*>(sm.PS);
    const float nw = reinterpret_cast<const float*>(reinterpret_cast<const unsigned char*>(sm.PS) +
                                                    TM * DV * sizeof(InT))[row];
#pragma unroll
    for (int tt = 0; tt < TM / 2; ++tt) {
        const int t = (TM / 2) * (tid >> 7) + tt;
        const float z = (t < T) ? to_f(zs[t * DV + row]) : 0.f;
        gz[tt] = nw * __fdividef(z, 1.f + __expf(-z));
    }
}

// PRE: commit-on-next-verify (the previous block's stash is applied to the state first).
// NORM: gated RMS normalisation of the outputs before they are stored.
template <typename InT, typename OutT, bool PRE, bool NORM>
__global__ void __launch_bounds__(kThreads, 2)
    gdn_verify_tc_kernel(const __grid_constant__ CUtensorMap smap, const VerifyArgs p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    TcSmem& sm = *reinterpret_cast<TcSmem*>(smem_raw);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int T = p.T;
    const int item = blockIdx.x;
    const int h = item % p.Hv;
    const int b = item / p.Hv;
    const int g = h / (p.Hv / p.Hk);
    const size_t head = (size_t)item;
    const size_t tok_stride = (size_t)p.Hv * DV;               // between tokens in v and o
    const size_t vo_base = ((size_t)b * T * p.Hv + h) * DV;    // token 0, row 0 of this head

    if ((smem_u32(smem_raw) & 1023u) != 0) {   // the swizzled tiles need 1024-byte alignment
        if (tid == 0 && p.status_word) atomicOr(p.status_word, kStatusWaitTimeout);
        return;
    }

    // 0. Every global load the CTA makes is issued here, before any arithmetic waits on one
    // (they are dependent round trips otherwise): the 64 KB state tile first, then the small
    // per-token loads.
    // Commit-on-next-verify: the previous block's stash for this head (one bulk copy, beside
    // the state tile) and its accept count L'.
    constexpr bool precommit = PRE;
    if (tid == 128) {
        mbar_init(&sm.full, 1);
        mbar_init(&sm.mma_done, 1);
        if (precommit || NORM) mbar_init(&sm.prev_full, 1);
        fence_barrier_init();
        mbar_arrive_expect_tx(&sm.full, kTileBytes);
        for (int kb = 0; kb < 4; ++kb) tc::tma_load_2d(&sm.S[kb * DV * 32], &smap, kb * 32, item * DV, &sm.full);
        if (precommit) {
            const size_t nf = stash_floats_per_head(p.prev_T, DK, DV);   // a multiple of 4 floats
            mbar_arrive_expect_tx(&sm.prev_full, (uint32_t)(nf * sizeof(float)));
            bulk_g2s(sm.PS, p.prev_stash + (size_t)item * nf, (uint32_t)(nf * sizeof(float)), &sm.prev_full);
        }
    }
    float a_in = 0.f, b_in = 0.f, alog = 0.f, dtb = 0.f;
    int L_in = 0, Lp_in = 0;
    if (warp == 0) {   // gate inputs (lane t = token t) and the accept counts
        if (lane < T) {
            const size_t gi = ((size_t)b * T + lane) * p.Hv + h;
            a_in = ld_in<InT>(p.a, gi);
            b_in = ld_in<InT>(p.b, gi);
        }
        alog = p.A_log[h];
        dtb = p.dt_bias[h];
        if (lane == 0 && !p.always_commit && p.accept_len) L_in = p.accept_len[b];
        if (precommit && lane == 1) Lp_in = p.prev_accept_len[b];
    }
    // khat_t, qhat_t (16 lanes per vector, 8 columns per lane) and the per-row v_t (row
    // tid % 128: threads tid and tid + 128 share a row and split its outputs).
    const int c16 = tid & 15;
    const int nrow = tid >> 4;               // 0..15 = NB rows
    const bool isq = nrow >= TM;
    const int tq = isq ? nrow - TM : nrow;
    const bool live = tq < T;
    float x[8];
    if (live) {
        ld8<InT>(isq ? p.q : p.k, (((size_t)b * T + tq) * p.Hk + g) * DK + 8 * c16, x);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = 0.f;
    }
    float vrow[TM];
#pragma unroll
    for (int t = 0; t < TM; ++t)
        vrow[t] = (t < T) ? ld_in<InT>(p.v, vo_base + t * tok_stride + (tid & (DV - 1))) : 0.f;
    float gz[TM / 2];   // gated norm: nw silu(z) of this row for its 4 tokens, formed in slack time
    if (warp == 4) {   // tensor memory: one allocation, off the gate chain
        if (lane == 0) {
            sm.fail = 0;
            sm.pfail = 0;
        }
        tc::tmem_alloc(&sm.tmem, 256);
        tc::tmem_relinquish();
    }
    // The CTA one resident wave ahead will find its state and per-token inputs in L2: without
    // this, every CTA starts by waiting on DRAM reads and the SM's two CTAs often wait at the
    // same time.
    if (p.prefetch_ahead > 0 && item + p.prefetch_ahead < (int)gridDim.x) {
        const int nx = item + p.prefetch_ahead;
        const int nh = nx % p.Hv, nb = nx / p.Hv, ng = nh / (p.Hv / p.Hk);
        const size_t el = p.in_bf16 ? 2 : 4;
        // Only whole rows of the state, q, k and v: each lies inside its array.
        if (tid == 32) bulk_prefetch_l2(p.state_in + (size_t)nx * DV * DK, kTileBytes);
        if (tid == 33 && p.prev_stash) {
            const size_t nf = stash_floats_per_head(p.prev_T, DK, DV);   // a multiple of 4 floats
            bulk_prefetch_l2(p.prev_stash + (size_t)nx * nf, (uint32_t)(nf * sizeof(float)));
        }
        if (tid >= 64 && tid < 64 + T) {   // one token of q, k and v per thread
            const int t = tid - 64;
            const char* qb = static_cast<const char*>(p.q);
            const char* kb = static_cast<const char*>(p.k);
            const char* vb = static_cast<const char*>(p.v);
            bulk_prefetch_l2(qb + ((((size_t)nb * T + t) * p.Hk + ng) * DK) * el, (uint32_t)(DK * el));
            bulk_prefetch_l2(kb + ((((size_t)nb * T + t) * p.Hk + ng) * DK) * el, (uint32_t)(DK * el));
            bulk_prefetch_l2(vb + ((((size_t)nb * T + t) * p.Hv + nh) * DV) * el, (uint32_t)(DV * el));
            if (NORM)   // the gate rows (v's layout)
                bulk_prefetch_l2(static_cast<const char*>(p.norm_z) + ((((size_t)nb * T + t) * p.Hv + nh) * DV) * el,
                                 (uint32_t)(DV * el));
        }
    }

    // 1b. Gates and the inclusive prefix sum of log-decays (warp 0, lane t = token t).
    if (warp == 0) {
        float gl = 0.f, be = 0.f;
        if (lane < T) {
            gl = -expf(alog) * softplus_f(a_in + dtb);
            be = 1.f / (1.f + expf(-b_in));
        }
        float Gs = gl;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(kFull, Gs, off);
            if (lane >= off) Gs += y;
        }
        if (lane < TM) {
            sm.G[lane] = Gs;
            sm.Beta[lane] = be;
            sm.D[lane] = (lane < T) ? expf(Gs) : 0.f;
        }
        if (lane == 0) {
            int L;
            if (p.always_commit) {
                L = T;
            } else if (p.accept_len) {
                L = L_in;
                if (L < 0 || L > T) {
                    if (p.status_word && h == 0) atomicOr(p.status_word, kStatusBadAccept);
                    L = -1;
                }
            } else {
                L = -2;
            }
            sm.L = L;
        }
        if (precommit && lane == 1) {
            int Lp = Lp_in;
            if (Lp < 0 || Lp > p.prev_T) {
                if (p.status_word && h == 0) atomicOr(p.status_word, kStatusBadAccept);
                Lp = 0;
            }
            sm.PL = Lp;
        }
    }

    // 1a. Normalised khat_t, qhat_t: plain copy + the split B tiles of the MMA; each thread
    // keeps its 8 normalised values for the Gram.
    float yv[8];
    {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
        ss = group_sum<16>(ss);
        const float inv = live ? (isq ? p.scale : 1.f) / sqrtf(ss + p.l2_eps) : 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float4 y, hi, lo;
            y = make_float4(x[4 * half] * inv, x[4 * half + 1] * inv, x[4 * half + 2] * inv, x[4 * half + 3] * inv);
            yv[4 * half] = y.x;
            yv[4 * half + 1] = y.y;
            yv[4 * half + 2] = y.z;
            yv[4 * half + 3] = y.w;
            hi = make_float4(tc::tf32_hi(y.x), tc::tf32_hi(y.y), tc::tf32_hi(y.z), tc::tf32_hi(y.w));
            lo = make_float4(y.x - hi.x, y.y - hi.y, y.z - hi.z, y.w - hi.w);
            *reinterpret_cast<float4*>(&sm.B2[tc::sw128_offset(nrow, 8 * c16 + 4 * half, 2 * NB) / 4]) = hi;
            *reinterpret_cast<float4*>(&sm.B2[tc::sw128_offset(NB + nrow, 8 * c16 + 4 * half, 2 * NB) / 4]) = lo;
            *reinterpret_cast<float4*>(&sm.KQ[nrow][8 * c16 + 4 * half]) = y;
        }
    }
    tc::fence_proxy_async_smem();   // the tensor core will read the B tiles written above
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem_a = sm.tmem, tmem_d = sm.tmem + 128;

    // 2g. Gram rows [Khat; Qhat] Khat^T, all threads, before the split and the MMAs (which
    // slow it down several-fold when they run alongside): thread (row n, lane c16) dots its 8
    // normalised columns (registers) with those of each khat_s, the row's 16 lanes reduce them
    // (halving butterfly), and lane 2s keeps entry s. Warps 4..7 only arrive at barrier 3.
    {
        float part[TM];
#pragma unroll
        for (int s = 0; s < TM; ++s) {
            const float4 k0 = *reinterpret_cast<const float4*>(&sm.KQ[s][8 * c16]);
            const float4 k1 = *reinterpret_cast<const float4*>(&sm.KQ[s][8 * c16 + 4]);
            float d = yv[0] * k0.x;
            d = fmaf(yv[1], k0.y, d);
            d = fmaf(yv[2], k0.z, d);
            d = fmaf(yv[3], k0.w, d);
            d = fmaf(yv[4], k1.x, d);
            d = fmaf(yv[5], k1.y, d);
            d = fmaf(yv[6], k1.z, d);
            part[s] = fmaf(yv[7], k1.w, d);
        }
        Halve<TM, 8>::run(part, c16);
        if ((c16 & 1) == 0) sm.Gram[nrow][c16 >> 1] = part[0];
    }

    if (warp >= 4) {
        named_arrive(3, 256);   // Gram rows 8..15 are stored
        // 2s. Warps 4..7 (the longest path): S_lo = S - trunc_tf32(S) into tensor memory (warp w owns lanes
        // 32 (w - 4) .. +31, i.e. those state rows, all 128 columns).
        const int q4 = warp - 4;
        const int row = 32 * q4 + lane;
        if (!mbar_wait_bounded(&sm.full, 0, kMaxPolls)) sm.fail = 1;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            float v[32];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 xs =
                    *reinterpret_cast<const float4*>(&sm.S[(cb * DV * 128 + row * 128 + ((q ^ (row & 7)) << 4)) / 4]);
                v[4 * q + 0] = xs.x - tc::tf32_hi(xs.x);
                v[4 * q + 1] = xs.y - tc::tf32_hi(xs.y);
                v[4 * q + 2] = xs.z - tc::tf32_hi(xs.z);
                v[4 * q + 3] = xs.w - tc::tf32_hi(xs.w);
            }
            tc::tmem_st32(tmem_a + ((uint32_t)(32 * q4) << 16) + 32 * cb, v);
        }
        tc::fence_before_sync();
        named_sync(2, 128);
        tc::fence_after_sync();
        // Then one thread issues the three tf32 passes: S (smem) B_hi + S (smem) B_lo +
        // S_lo (tmem) B_hi.
        if (tid == 128 && !sm.fail) {
            // Columns 0..15 accumulate S B_hi + S_lo B_hi, columns 16..31 S B_lo.
            const uint32_t id32 = tc::idesc_tf32(DV, 2 * NB), id16 = tc::idesc_tf32(DV, NB);
            const uint32_t as = smem_u32(sm.S);
            const uint32_t bb = smem_u32(sm.B2);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_tf32_ss(tmem_d, tc::desc_kmajor_sw128(as + kb * DV * 128 + ks * 32),
                                    tc::desc_kmajor_sw128(bb + kb * 2 * NB * 128 + ks * 32), id32, kb + ks > 0);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_tf32_ts(tmem_d, tmem_a + kb * 32 + ks * 8,
                                    tc::desc_kmajor_sw128(bb + kb * 2 * NB * 128 + ks * 32), id16, true);
            tc::mma_commit(&sm.mma_done);
        }
        if (NORM) gate_factors<InT>(sm, p, T, tid, gz);   // tokens 4..7, while the MMAs run
    } else {
        if (NORM && warp == 3) {
            // The block's gate rows and the weights into PS (needed only by the last phase): lane
            // 0 posts the bytes, lanes 0..T-1 copy a row each, lane T the weights. Off the split's
            // path, after the block barrier that follows the barrier's initialisation.
            const uint32_t row_bytes = DV * sizeof(InT);
            if (lane == 0) mbar_arrive_expect_tx(&sm.prev_full, T * row_bytes + DV * 4);
            __syncwarp();
            if (lane < T)
                bulk_g2s(reinterpret_cast<unsigned char*>(sm.PS) + lane * row_bytes,
                         static_cast<const InT*>(p.norm_z) + vo_base + lane * tok_stride, row_bytes, &sm.prev_full);
            else if (lane == T)
                bulk_g2s(reinterpret_cast<unsigned char*>(sm.PS) + TM * row_bytes, p.norm_w, DV * 4, &sm.prev_full);
        }
        named_sync(3, 256);     // all 16 Gram rows are stored
        // ... the T x T algebra (barrier 1 between steps): the decayed coefficients, one entry
        // per thread, and the commit decays ...
        const int Lc = sm.L;
        if (precommit) {
            if (!mbar_wait_bounded(&sm.prev_full, 0, kMaxPolls)) sm.pfail = 1;
            const int Lp = sm.PL;
            const float* pg = &sm.PS[p.prev_T * DK];   // the previous block's cumulative log-decays
            const float glast = (Lp > 0) ? pg[Lp - 1] : 0.f;
#pragma unroll
            for (int t = 0; t < TM; ++t)
                if (t < Lp) sm.PS[t * DK + tid] *= expf(glast - pg[t]);
            if (tid == 0) sm.PD = (Lp > 0) ? expf(glast) : 1.f;
        }
        if (tid < TM * TM) {
            const int t = tid / TM, s = tid % TM;
            const bool inq = t < T && s <= t;
            const float dec = inq ? expf(sm.G[t] - sm.G[s]) : 0.f;
            sm.A[t][s] = (inq && s < t) ? sm.Beta[t] * dec * sm.Gram[t][s] : 0.f;
            sm.Cq[t][s] = inq ? dec * sm.Gram[TM + t][s] : 0.f;
        } else if (tid < TM * TM + TM) {
            const int t = tid - TM * TM;
            sm.Ec[t] = (Lc > 0 && t < Lc) ? expf(sm.G[Lc - 1] - sm.G[t]) : 0.f;
        }
        named_sync(1, 128);
        // ... the unit-triangular inverse Tm = (I + A)^-1 by forward substitution (warp 0, lane
        // s = column s, A read once into registers) ...
        if (warp == 0 && lane < TM) {
            const int s = lane;
            float a[TM][TM];
#pragma unroll
            for (int t = 0; t < TM; ++t)
#pragma unroll
                for (int m = 0; m < TM; m += 4) {
                    const float4 v4 = *reinterpret_cast<const float4*>(&sm.A[t][m]);
                    a[t][m] = v4.x;
                    a[t][m + 1] = v4.y;
                    a[t][m + 2] = v4.z;
                    a[t][m + 3] = v4.w;
                }
            float col[TM];
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                float x = (t == s) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < t; ++m) x = fmaf(-a[t][m], col[m], x);
                col[t] = (t >= s) ? x : 0.f;
                sm.Tm[t][s] = col[t];
            }
        }
        named_sync(1, 128);
        // ... the output and commit coefficients Mo = Cq Tm, E[t][s] = Ec[t] Tm[t][s] (one
        // entry per thread) ...
        if (tid < TM * TM) {
            const int t = tid / TM, s = tid % TM;
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < TM; ++m)
                if (m >= s && m <= t) acc = fmaf(sm.Cq[t][m], sm.Tm[m][s], acc);
            sm.Mo[t][s] = (s <= t) ? acc : 0.f;
        } else {
            const int e = tid - TM * TM;
            const int t = e / TM, s = e % TM;
            sm.E[t][s] = (s <= t) ? sm.Ec[t] * sm.Tm[t][s] : 0.f;
        }
        if (tid == 0) sm.DL = (Lc > 0) ? sm.D[Lc - 1] : 1.f;
        named_sync(1, 128);
        // ... and Keff_s = sum_t E[t][s] khat_t (warps 0..3, column j = tid, 8 entries each).
        if (Lc > 0) {
#pragma unroll
            for (int s = 0; s < TM; ++s) {
                float acc = 0.f;
#pragma unroll
                for (int t = 0; t < TM; ++t) acc = fmaf(sm.E[t][s], sm.KQ[t][tid], acc);
                sm.Keff[s][tid] = acc;
            }
        }
        if (precommit) {
            // ... and W[t][n] = KP_t . [khat; qhat]_n (one entry per thread; rotated columns, so
            // the 8 threads of a quarter-warp read 8 different bank groups).
            const int t = tid >> 4, n = tid & (NB - 1);
            float acc = 0.f;
            if (t < sm.PL) {
#pragma unroll 8
                for (int c = 0; c < DK / 4; ++c) {
                    const int cc = (c + n) & (DK / 4 - 1);
                    const float4 kp = *reinterpret_cast<const float4*>(&sm.PS[t * DK + 4 * cc]);
                    const float4 kq = *reinterpret_cast<const float4*>(&sm.KQ[n][4 * cc]);
                    acc = fmaf(kp.x, kq.x, acc);
                    acc = fmaf(kp.y, kq.y, acc);
                    acc = fmaf(kp.z, kq.z, acc);
                    acc = fmaf(kp.w, kq.w, acc);
                }
            }
            sm.W[t][n] = acc;
        }
        if (NORM) gate_factors<InT>(sm, p, T, tid, gz);   // tokens 0..3 (a shorter path than the split's)
    }
    __syncthreads();
    const int L = sm.L;
    bool ok = !sm.fail && !sm.pfail;
    const int off_pu = p.prev_T * DK + ((p.prev_T + 3) & ~3);   // u' rows in PS

    // 3. Row tid % 128 (TMEM lane): the dots from tensor memory and x_s (both halves of the
    // block), then the outputs and stash of tokens 4 half .. +3 (half = tid / 128); threads
    // 0..127 keep x for the commit.
    if (ok && !mbar_wait_bounded(&sm.mma_done, 0, kMaxPolls)) ok = false;
    tc::fence_after_sync();
    {
        const int row = tid & (DV - 1);
        const int hb = tid >> 7;
        float dots[16], dlo[16];
        tc::tmem_ld16(tmem_d + ((uint32_t)(32 * (warp & 3)) << 16), dots);
        tc::tmem_ld16(tmem_d + ((uint32_t)(32 * (warp & 3)) << 16) + 16, dlo);
#pragma unroll
        for (int i = 0; i < 16; ++i) dots[i] += dlo[i];
        if (precommit) {
            const float pd = sm.PD;
            const int Lp = sm.PL;
#pragma unroll
            for (int i = 0; i < 16; ++i) dots[i] *= pd;
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                if (t < Lp) {
                    const float u = sm.PS[off_pu + t * DV + row];
#pragma unroll
                    for (int i = 0; i < 16; ++i) dots[i] = fmaf(u, sm.W[t][i], dots[i]);
                }
            }
        }
        float xs[TM];
#pragma unroll
        for (int s = 0; s < TM; ++s) xs[s] = sm.Beta[s] * (vrow[s] - sm.D[s] * dots[s]);
        if (hb == 0) {
#pragma unroll
            for (int s = 0; s < TM; s += 2)
                *reinterpret_cast<float4*>(&sm.X2[row][s]) = make_float4(xs[s], xs[s], xs[s + 1], xs[s + 1]);
        }
        // Outputs of tokens 4 hb .. 4 hb + 3 for this row (0 past T).
        float ovs[TM / 2];
#pragma unroll
        for (int tt = 0; tt < TM / 2; ++tt) {
            const int t = (TM / 2) * hb + tt;
            float ov = 0.f;
            if (t < T) {
                ov = sm.D[t] * (hb ? dots[TM + TM / 2 + tt] : dots[TM + tt]);   // static indices
#pragma unroll
                for (int s = 0; s < TM; ++s)
                    if (s <= t) ov = fmaf(sm.Mo[t][s], xs[s], ov);
            }
            ovs[tt] = ov;
        }
        if (NORM) {
            // Each token's 128 outputs sit in the 128 threads of this half (warps 4 hb .. +3):
            // the warp's four sums of squares by a halving butterfly (token tt ends in lanes
            // 8 tt .. 8 tt + 7), then the half's four partials (named barrier 5 + hb, which every
            // thread of the half reaches whatever ok is).
            float sq[TM / 2];
#pragma unroll
            for (int tt = 0; tt < TM / 2; ++tt) sq[tt] = ovs[tt] * ovs[tt];
            Halve<TM / 2, 16>::run(sq, lane);
            if ((lane & 7) == 0) sm.NSS[warp][lane >> 3] = sq[0];
            named_sync(5 + hb, 128);
#pragma unroll
            for (int tt = 0; tt < TM / 2; ++tt) {
                const float tot = sm.NSS[4 * hb][tt] + sm.NSS[4 * hb + 1][tt] + sm.NSS[4 * hb + 2][tt] +
                                  sm.NSS[4 * hb + 3][tt];
                ovs[tt] *= rsqrtf(tot / (float)DV + p.norm_eps) * gz[tt];
            }
        }
        if (ok) {
            OutT* op = reinterpret_cast<OutT*>(p.o);
#pragma unroll
            for (int tt = 0; tt < TM / 2; ++tt) {
                const int t = (TM / 2) * hb + tt;
                if (t < T) st_out<OutT>(op, vo_base + t * tok_stride + row, ovs[tt]);
            }
            if (p.stash) {
                float* st = p.stash + head * stash_floats_per_head(T, DK, DV);
                const size_t off_u = (size_t)T * DK + (((size_t)T + 3) & ~size_t(3));
#pragma unroll
                for (int tt = 0; tt < TM / 2; ++tt) {
                    const int t = (TM / 2) * hb + tt;
                    if (t < T) {
                        float u = 0.f;
#pragma unroll
                        for (int s = 0; s < TM; ++s)
                            if (s <= t) u = fmaf(sm.Tm[t][s], xs[s], u);
                        st[off_u + (size_t)t * DV + row] = u;
                    }
                }
                for (int e = tid; e < T * DK; e += kThreads) st[e] = sm.KQ[e / DK][e % DK];
                if (tid < T) st[(size_t)T * DK + tid] = sm.G[tid];
            }
        }
    }
    tc::fence_before_sync();
    ok = !__syncthreads_or(!ok);
    if (!ok && tid == 0 && p.status_word) atomicOr(p.status_word, kStatusWaitTimeout);

    // 4. Commit at L (rollback / bad L: the initial state, skipped when in place).
    // After a commit-on-next-verify the state is always written: S' committed at this block's
    // L, or S' itself (no accept counts: the new base for the next call; rollback; bad L).
    const bool write_state = precommit || (L != -2 && !(L <= 0 && p.state_out == p.state_in));
    if (ok && write_state) {
        float* dst = p.state_out + head * (size_t)DV * DK;
        const float dl = sm.DL;
        const int Lp = precommit ? sm.PL : 0;
        const float pd = precommit ? sm.PD : 1.f;
        switch (L > 0 ? L : 0) {
            case 1: commit_rows<1, PRE>(sm, dst, warp, lane, dl, Lp, pd, off_pu); break;
            case 2: commit_rows<2, PRE>(sm, dst, warp, lane, dl, Lp, pd, off_pu); break;
            case 3: commit_rows<3, PRE>(sm, dst, warp, lane, dl, Lp, pd, off_pu); break;
            case 4: commit_rows<4, PRE>(sm, dst, warp, lane, dl, Lp, pd, off_pu); break;
            case 5: commit_rows<5, PRE>(sm, dst, warp, lane, dl, Lp, pd, off_pu); break;
            case 6: commit_rows<6, PRE>(sm, dst, warp, lane, dl, Lp, pd, off_pu); break;
            case 7: commit_rows<7, PRE>(sm, dst, warp, lane, dl, Lp, pd, off_pu); break;
            case 8: commit_rows<8, PRE>(sm, dst, warp, lane, dl, Lp, pd, off_pu); break;
            default: commit_rows<0, PRE>(sm, dst, warp, lane, dl, Lp, pd, off_pu); break;
        }
    }

    // Drain after a timeout (bounded), then free the tensor memory (always).
    if (!ok && tid == 0) {
        mbar_wait_bounded(&sm.full, 0, kMaxPolls);
        if (precommit || NORM) mbar_wait_bounded(&sm.prev_full, 0, kMaxPolls);
        if (!sm.fail) mbar_wait_bounded(&sm.mma_done, 0, kMaxPolls);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 4) tc::tmem_dealloc(tmem_a, 256);
}

template <typename InT, typename OutT, bool PRE, bool NORM>
cudaError_t launch_tc_t(const VerifyArgs& a, cudaStream_t stream) {
    constexpr size_t smem = sizeof(TcSmem);
    cudaError_t e = ensure_smem_attr<gdn_verify_tc_kernel<InT, OutT, PRE, NORM>>((int)smem);
    if (e != cudaSuccess) return e;
    CUtensorMap map;
    e = tc::encode_tmap_f32_sw128(&map, a.state_in, (uint64_t)a.B * a.Hv * DV, DK, DV);
    if (e != cudaSuccess) return e;
    int nsm = 0;
    e = current_sm_count(&nsm);
    if (e != cudaSuccess) return e;
    VerifyArgs ap = a;
    ap.prefetch_ahead = 2 * nsm;   // two CTAs per SM are resident
    gdn_verify_tc_kernel<InT, OutT, PRE, NORM><<<a.B * a.Hv, kThreads, smem, stream>>>(map, ap);
    return cudaGetLastError();
}

template <typename InT, typename OutT>
cudaError_t launch_tc_pre(const VerifyArgs& a, cudaStream_t stream) {
    if (a.prev_stash) return launch_tc_t<InT, OutT, true, false>(a, stream);
    return a.norm_z ? launch_tc_t<InT, OutT, false, true>(a, stream) : launch_tc_t<InT, OutT, false, false>(a, stream);
}

}  // namespace

bool tc_kernel_applies(const VerifyArgs& a, int num_sms) {
    // Single-token decode stays on the CUDA-core head kernel (measured faster there).
    return a.dk == DK && a.dv == DV && a.T >= 2 && a.T <= TM && (long long)a.B * a.Hv >= num_sms;
}

cudaError_t launch_verify_tc(const VerifyArgs& a, cudaStream_t stream) {
    if (a.in_bf16)
        return a.out_bf16 ? launch_tc_pre<__nv_bfloat16, __nv_bfloat16>(a, stream)
                          : launch_tc_pre<__nv_bfloat16, float>(a, stream);
    return a.out_bf16 ? launch_tc_pre<float, __nv_bfloat16>(a, stream) : launch_tc_pre<float, float>(a, stream);
}

}  // namespace gdn
