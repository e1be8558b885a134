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
//     state-independent part (normalised keys / queries, the Gram matrix on the tensor cores,
//     the triangular inverse, Mo and Keff on the CUDA cores), written to the workspace;
//   gdn_prefill_scan_kernel, one CTA per (sequence, value head), chunk after chunk: the state
//     lives in tensor memory (fp32) as the A operand of P | R and the accumulator of the
//     update; Mo and Keff^T of the next chunk arrive by TMA while the current one runs.
// Precision (kind::tf32 reads operands as truncated tf32): the state dots and the Gram take
// one tf32 pass; X Mo^T and X Keff take three (X_hi B_hi + X_hi B_lo + X_lo B_hi), which an
// fp32 emulation of this exact algorithm against the fp64 recurrence put at ~8e-4 relative
// error at worst, against ~1.5e-3 for one pass everywhere.
// Every mbarrier wait is bounded; a timeout sets GDN_STATUS_WAIT_TIMEOUT and the CTA stops
// writing, drains what it issued (bounded) and frees its tensor memory.
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
constexpr int kThreads = 256;
constexpr uint32_t kMaxPolls = 1u << 24;

// Workspace record of one (sequence, value head, chunk), fp32:
//   Mo     [64 t][64 s]      (row-major: s contiguous; the scan's B operand, K-major)
//   KeffT  [128 j][64 s]     (row-major: s contiguous; the scan's B operand, K-major)
//   vec    d[64], beta[64], d_C, pad to 144 floats
constexpr size_t kMoFloats = kC * kC;
constexpr size_t kKeFloats = DK * kC;
constexpr size_t kVecFloats = 144;

__host__ __device__ inline size_t n_chunks_of(int T) { return ((size_t)T + kC - 1) / kC; }

// ---------------------------------------------------------------- prep kernel

struct __align__(1024) PrepSmem {
    float KQ[2 * kC * DK];     // [khat; qhat] rows, SW128 K-major (4 blocks of [128 rows][32])
    float Kk[kC][kC];          // Gram rows, then A in place
    float Qk[kC][kC];          // then Cq in place
    float Tm[kC][kC];
    float G[kC], Beta[kC], Dd[kC], Ec[kC];
    uint64_t mma_done;
    uint32_t tmem;
};

template <typename InT>
__global__ void __launch_bounds__(kThreads, 2)
    gdn_prefill_prep_kernel(const VerifyArgs p, float* __restrict__ ws_mo, float* __restrict__ ws_ke,
                            float* __restrict__ ws_vec) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    PrepSmem& sm = *reinterpret_cast<PrepSmem*>(smem_raw);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int c = blockIdx.x;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int T = p.T;
    const int g = h / (p.Hv / p.Hk);
    const int t0 = c * kC;
    const int n = min(kC, T - t0);   // tokens in this chunk
    const size_t unit = ((size_t)b * p.Hv + h) * n_chunks_of(T) + c;

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

    // 1. khat / qhat rows (16 lanes x 8 columns per row, 2 rows per pass of 256 threads ...)
    for (int r0 = 0; r0 < 2 * kC; r0 += kThreads / 16) {
        const int r = r0 + (tid >> 4);       // 0..127: rows 0..63 khat, 64..127 qhat
        const int c16 = tid & 15;
        const bool isq = r >= kC;
        const int t = isq ? r - kC : r;
        const bool live = t < n;
        float x[8];
        if (live) {
            ld8<InT>(isq ? p.q : p.k, (((size_t)b * T + t0 + t) * p.Hk + g) * DK + 8 * c16, x);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = 0.f;
        }
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
        ss = group_sum<16>(ss);
        const float inv = live ? (isq ? p.scale : 1.f) / sqrtf(ss + p.l2_eps) : 0.f;
        *reinterpret_cast<float4*>(&sm.KQ[tc::sw128_offset(r, 8 * c16, 2 * kC) / 4]) =
            make_float4(x[0] * inv, x[1] * inv, x[2] * inv, x[3] * inv);
        *reinterpret_cast<float4*>(&sm.KQ[tc::sw128_offset(r, 8 * c16 + 4, 2 * kC) / 4]) =
            make_float4(x[4] * inv, x[5] * inv, x[6] * inv, x[7] * inv);
    }
    // Gates and the inclusive prefix sum of log-decays over the chunk (warps 0, 1: 64 lanes).
    if (warp < 2) {
        const int t = tid;                   // 0..63
        float gl = 0.f, be = 0.f;
        if (t < n) {
            const size_t gi = ((size_t)b * T + t0 + t) * p.Hv + h;
            gl = -expf(p.A_log[h]) * softplus_f(ld_in<InT>(p.a, gi) + p.dt_bias[h]);
            be = 1.f / (1.f + expf(-ld_in<InT>(p.b, gi)));
        }
        float Gs = gl;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(kFull, Gs, off);
            if (lane >= off) Gs += y;
        }
        sm.G[t] = Gs;                        // warp 1 adds warp 0's total below
        sm.Beta[t] = be;
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem;

    // 2. Gram on the tensor cores: D (128 x 64) = [Khat; Qhat] Khat^T, one tf32 pass.
    if (tid == 0) {
        const uint32_t id = tc::idesc_tf32(2 * kC, kC);
        const uint32_t kq = smem_u32(sm.KQ);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint32_t off = kb * (2 * kC) * 128 + ks * 32;
                tc::mma_tf32_ss(tmem, tc::desc_kmajor_sw128(kq + off), tc::desc_kmajor_sw128(kq + off), id,
                                kb + ks > 0);
            }
        tc::mma_commit(&sm.mma_done);
    }
    // Meanwhile: finish the prefix sum across the two warps, and the decay vectors.
    if (warp == 1) sm.G[tid] += sm.G[31];
    __syncthreads();
    if (tid < kC) {
        const float GC = sm.G[n - 1];
        sm.Dd[tid] = (tid < n) ? expf(sm.G[tid]) : 0.f;
        sm.Ec[tid] = (tid < n) ? expf(GC - sm.G[tid]) : 0.f;
    }
    bool ok = mbar_wait_bounded(&sm.mma_done, 0, kMaxPolls);
    tc::fence_after_sync();
    if (warp < 4) {
        // Lane r of warp w holds Gram row 32 w + r: rows 0..63 are Kk, 64..127 Qk.
        const int r = 32 * warp + lane;
        float (*dst)[kC] = r < kC ? sm.Kk : sm.Qk;
        const int rr = r & (kC - 1);
#pragma unroll
        for (int cb = 0; cb < kC; cb += 16) {
            float v[16];
            tc::tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + cb, v);
#pragma unroll
            for (int e = 0; e < 16; ++e) dst[rr][cb + e] = v[e];
        }
    }
    tc::fence_before_sync();
    __syncthreads();

    // 3. A (strictly lower, in Kk) and Cq (lower with diagonal, in Qk); decays as exp of differences.
    for (int e = tid; e < kC * kC; e += kThreads) {
        const int t = e >> 6, s = e & (kC - 1);
        const bool inq = t < n && s <= t;
        const float dec = inq ? expf(sm.G[t] - sm.G[s]) : 0.f;
        sm.Kk[t][s] = (inq && s < t) ? sm.Beta[t] * dec * sm.Kk[t][s] : 0.f;
        sm.Qk[t][s] = inq ? dec * sm.Qk[t][s] : 0.f;
    }
    __syncthreads();

    // 4. Tm = (I + A)^-1 by forward substitution, one column per thread (threads 0..63).
    if (tid < kC) {
        const int s = tid;
        for (int t = 0; t < kC; ++t) {
            float x = (t == s) ? 1.f : 0.f;
            if (t > s) {
                float acc = 0.f;
                for (int m = s; m < t; ++m) acc = fmaf(sm.Kk[t][m], sm.Tm[m][s], acc);
                x = -acc;
            }
            sm.Tm[t][s] = (t >= s) ? x : 0.f;
        }
    }
    __syncthreads();

    // 5. Mo = Cq Tm (lower triangular) straight to the workspace, and the vectors.
    {
        float* mo = ws_mo + unit * kMoFloats;
        for (int e = tid; e < kC * kC; e += kThreads) {
            const int t = e >> 6, s = e & (kC - 1);
            float acc = 0.f;
            for (int m = s; m <= t; ++m) acc = fmaf(sm.Qk[t][m], sm.Tm[m][s], acc);
            mo[e] = (s <= t) ? acc : 0.f;
        }
        float* vec = ws_vec + unit * kVecFloats;
        if (tid < kC) {
            vec[tid] = sm.Dd[tid];
            vec[kC + tid] = sm.Beta[tid];
        }
        if (tid == 0) vec[2 * kC] = expf(sm.G[n - 1]);
    }

    // 6. Keff^T[j][s] = sum_{t >= s} khat_t[j] exp(G_C - G_t) Tm[t][s]: column j = tid % 128,
    // s in one half per thread.
    {
        const int j = tid & (DK - 1);
        const int s0 = (tid >> 7) * (kC / 2);
        float kt[kC];
#pragma unroll
        for (int t = 0; t < kC; ++t) kt[t] = sm.KQ[tc::sw128_offset(t, j, 2 * kC) / 4] * sm.Ec[t];
        float* ke = ws_ke + unit * kKeFloats + (size_t)j * kC;
        for (int s = s0; s < s0 + kC / 2; ++s) {
            float acc = 0.f;
#pragma unroll
            for (int t = 0; t < kC; ++t)
                if (t >= s) acc = fmaf(kt[t], sm.Tm[t][s], acc);
            ke[s] = acc;
        }
    }
    if (!ok && tid == 0 && p.status_word) atomicOr(p.status_word, kStatusWaitTimeout);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 64);
}

// ---------------------------------------------------------------- scan kernel


struct __align__(1024) ScanSmem {
    float KQ[2 * kC * DK];       // [khat; qhat] rows of the current chunk, SW128 K-major
    float Mo[2][kC * kC];        // TMA: [64 t][64 s] K-major SW128 (2 blocks of [64][32]), 2 buffers
    float MoLo[kC * kC];
    float Ke[2][DK * kC];        // TMA: [128 j][64 s] K-major SW128 (2 blocks of [128][32]), 2 buffers
    float KeLo[DK * kC];
    float Dd[kC], Beta[kC];
    float DC;
    uint64_t full[2];
    uint64_t mma1, mma2;
    uint32_t tmem;
};

// TMEM columns: S 0..127, P|R 128..255, O 256..319, X_hi 320..383, X_lo 384..447.
constexpr uint32_t kColS = 0, kColPR = 128, kColO = 256, kColXh = 320, kColXl = 384;

template <typename InT, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    gdn_prefill_scan_kernel(const __grid_constant__ CUtensorMap mo_map, const __grid_constant__ CUtensorMap ke_map,
                            const VerifyArgs p, const float* __restrict__ ws_vec) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    ScanSmem& sm = *reinterpret_cast<ScanSmem*>(smem_raw);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int q4 = warp & 3;               // tensor-memory quadrant of this warp
    const int h = blockIdx.x;
    const int b = blockIdx.y;
    const int T = p.T;
    const int g = h / (p.Hv / p.Hk);
    const int nch = (int)n_chunks_of(T);
    const size_t head = (size_t)b * p.Hv + h;
    const size_t unit0 = head * nch;
    constexpr uint32_t kMoBytes = kC * kC * 4, kKeBytes = DK * kC * 4;

    if ((smem_u32(smem_raw) & 1023u) != 0) {
        if (tid == 0 && p.status_word) atomicOr(p.status_word, kStatusWaitTimeout);
        return;
    }
    if (tid == 0) {
        mbar_init(&sm.full[0], 1);
        mbar_init(&sm.full[1], 1);
        mbar_init(&sm.mma1, 1);
        mbar_init(&sm.mma2, 1);
        fence_barrier_init();
        // chunks 0 and 1 of this head
        for (int i = 0; i < 2 && i < nch; ++i) {
            mbar_arrive_expect_tx(&sm.full[i], kMoBytes + kKeBytes);
            for (int kb = 0; kb < 2; ++kb) {
                tc::tma_load_2d(&sm.Mo[i][kb * kC * 32], &mo_map, kb * 32, (int)((unit0 + i) * kC), &sm.full[i]);
                tc::tma_load_2d(&sm.Ke[i][kb * DK * 32], &ke_map, kb * 32, (int)((unit0 + i) * DK), &sm.full[i]);
            }
        }
    }
    if (warp == 0) {
        tc::tmem_alloc(&sm.tmem, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem;
    const uint32_t lanebase = tmem + ((uint32_t)(32 * q4) << 16);
    const int row = 32 * q4 + lane;        // state row of this thread (warps w and w+4 share it)
    const int half = warp >> 2;            // which half of the columns this warp handles

    // Initial state into tensor memory (zero when state_in is NULL): columns 64*half .. +63.
    {
        const float* src = p.state_in ? p.state_in + (head * DV + row) * DK : nullptr;
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) {
            float v[32];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 x = src ? __ldg(reinterpret_cast<const float4*>(src + 64 * half + 32 * cb) + q)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                v[4 * q] = x.x;
                v[4 * q + 1] = x.y;
                v[4 * q + 2] = x.z;
                v[4 * q + 3] = x.w;
            }
            tc::tmem_st32(lanebase + kColS + 64 * half + 32 * cb, v);
        }
    }

    bool ok = true;
    for (int c = 0; c < nch; ++c) {
        const int buf = c & 1;
        const int t0 = c * kC;
        const int n = min(kC, T - t0);
        const size_t unit = unit0 + c;

        // a. khat / qhat rows of this chunk into the B tile (raw fp32; the MMA truncates).
        for (int r0 = 0; r0 < 2 * kC; r0 += kThreads / 16) {
            const int r = r0 + (tid >> 4);
            const int c16 = tid & 15;
            const bool isq = r >= kC;
            const int t = isq ? r - kC : r;
            const bool live = t < n;
            float x[8];
            if (live) {
                ld8<InT>(isq ? p.q : p.k, (((size_t)b * T + t0 + t) * p.Hk + g) * DK + 8 * c16, x);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = 0.f;
            }
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
            ss = group_sum<16>(ss);
            const float inv = live ? (isq ? p.scale : 1.f) / sqrtf(ss + p.l2_eps) : 0.f;
            *reinterpret_cast<float4*>(&sm.KQ[tc::sw128_offset(r, 8 * c16, 2 * kC) / 4]) =
                make_float4(x[0] * inv, x[1] * inv, x[2] * inv, x[3] * inv);
            *reinterpret_cast<float4*>(&sm.KQ[tc::sw128_offset(r, 8 * c16 + 4, 2 * kC) / 4]) =
                make_float4(x[4] * inv, x[5] * inv, x[6] * inv, x[7] * inv);
        }
        if (tid < kC) {
            const float* vec = ws_vec + unit * kVecFloats;
            sm.Dd[tid] = vec[tid];
            sm.Beta[tid] = vec[kC + tid];
            if (tid == 0) sm.DC = vec[2 * kC];
        }
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();

        // b. P | R = S [Khat; Qhat]^T (A = S in tensor memory, one tf32 pass).
        if (tid == 0) {
            const uint32_t id = tc::idesc_tf32(DV, 2 * kC);
            const uint32_t kq = smem_u32(sm.KQ);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_tf32_ts(tmem + kColPR, tmem + kColS + kb * 32 + ks * 8,
                                    tc::desc_kmajor_sw128(kq + kb * (2 * kC) * 128 + ks * 32), id, kb + ks > 0);
            tc::mma_commit(&sm.mma1);
        }

        // c. Meanwhile: this chunk's Mo and Keff^T (TMA) split into tf32 high / low parts.
        if (!mbar_wait_bounded(&sm.full[buf], (c >> 1) & 1, kMaxPolls)) ok = false;
        for (int e = tid * 4; e < kC * kC; e += kThreads * 4) {
            float4 x = *reinterpret_cast<const float4*>(&sm.Mo[buf][e]);
            const float4 hi = make_float4(tc::tf32_hi(x.x), tc::tf32_hi(x.y), tc::tf32_hi(x.z), tc::tf32_hi(x.w));
            *reinterpret_cast<float4*>(&sm.MoLo[e]) = make_float4(x.x - hi.x, x.y - hi.y, x.z - hi.z, x.w - hi.w);
        }
        for (int e = tid * 4; e < DK * kC; e += kThreads * 4) {
            float4 x = *reinterpret_cast<const float4*>(&sm.Ke[buf][e]);
            const float4 hi = make_float4(tc::tf32_hi(x.x), tc::tf32_hi(x.y), tc::tf32_hi(x.z), tc::tf32_hi(x.w));
            *reinterpret_cast<float4*>(&sm.KeLo[e]) = make_float4(x.x - hi.x, x.y - hi.y, x.z - hi.z, x.w - hi.w);
        }
        // v_s for this thread's row, tokens 32*half .. +31 (the X columns this warp forms).
        float vv[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int t = 32 * half + e;
            vv[e] = (t < n) ? ld_in<InT>(p.v, (((size_t)b * T + t0 + t) * p.Hv + h) * DV + row) : 0.f;
        }

        // d. X = beta (v - d P) into tensor memory (hi / lo), and S <- d_C S in place.
        if (!mbar_wait_bounded(&sm.mma1, c & 1, kMaxPolls)) ok = false;
        tc::fence_after_sync();
        {
            float pv[32], xh[32], xl[32];
            tc::tmem_ld16(lanebase + kColPR + 32 * half, *reinterpret_cast<float(*)[16]>(&pv[0]));
            tc::tmem_ld16(lanebase + kColPR + 32 * half + 16, *reinterpret_cast<float(*)[16]>(&pv[16]));
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int s = 32 * half + e;
                const float x = sm.Beta[s] * (vv[e] - sm.Dd[s] * pv[e]);
                xh[e] = tc::tf32_hi(x);
                xl[e] = x - xh[e];
            }
            tc::tmem_st32(lanebase + kColXh + 32 * half, xh);
            tc::tmem_st32(lanebase + kColXl + 32 * half, xl);
            const float dC = sm.DC;
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                float sv[32];
                tc::tmem_ld16(lanebase + kColS + 64 * half + 32 * cb, *reinterpret_cast<float(*)[16]>(&sv[0]));
                tc::tmem_ld16(lanebase + kColS + 64 * half + 32 * cb + 16, *reinterpret_cast<float(*)[16]>(&sv[16]));
#pragma unroll
                for (int e = 0; e < 32; ++e) sv[e] *= dC;
                tc::tmem_st32(lanebase + kColS + 64 * half + 32 * cb, sv);
            }
        }
        tc::fence_proxy_async_smem();   // MoLo / KeLo were written by the threads
        tc::fence_before_sync();
        ok = !__syncthreads_or(!ok);
        tc::fence_after_sync();
        if (!ok) break;

        // e. O = X Mo^T and S += X Keff, three passes each (A = X from tensor memory).
        if (tid == 0) {
            const uint32_t idO = tc::idesc_tf32(DV, kC), idS = tc::idesc_tf32(DV, DK);
            const uint32_t moh = smem_u32(sm.Mo[buf]), mol = smem_u32(sm.MoLo);
            const uint32_t keh = smem_u32(sm.Ke[buf]), kel = smem_u32(sm.KeLo);
#pragma unroll
            for (int pass = 0; pass < 3; ++pass) {
                const uint32_t xa = tmem + (pass == 2 ? kColXl : kColXh);
                const uint32_t mo = pass == 1 ? mol : moh;
                const uint32_t ke = pass == 1 ? kel : keh;
#pragma unroll
                for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint32_t ka = xa + kb * 32 + ks * 8;
                        tc::mma_tf32_ts(tmem + kColO, ka, tc::desc_kmajor_sw128(mo + kb * kC * 128 + ks * 32), idO,
                                        pass + kb + ks > 0);
                        tc::mma_tf32_ts(tmem + kColS, ka, tc::desc_kmajor_sw128(ke + kb * DK * 128 + ks * 32), idS,
                                        true);
                    }
            }
            tc::mma_commit(&sm.mma2);
        }
        if (!mbar_wait_bounded(&sm.mma2, c & 1, kMaxPolls)) ok = false;
        tc::fence_after_sync();

        // f. Outputs: o_t[row] = d_t R[row][t] + O[row][t], tokens 32*half .. +31.
        {
            float rv[32], ov[32];
            tc::tmem_ld16(lanebase + kColPR + kC + 32 * half, *reinterpret_cast<float(*)[16]>(&rv[0]));
            tc::tmem_ld16(lanebase + kColPR + kC + 32 * half + 16, *reinterpret_cast<float(*)[16]>(&rv[16]));
            tc::tmem_ld16(lanebase + kColO + 32 * half, *reinterpret_cast<float(*)[16]>(&ov[0]));
            tc::tmem_ld16(lanebase + kColO + 32 * half + 16, *reinterpret_cast<float(*)[16]>(&ov[16]));
            if (ok) {
                OutT* op = reinterpret_cast<OutT*>(p.o);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int t = 32 * half + e;
                    if (t < n)
                        st_out<OutT>(op, (((size_t)b * T + t0 + t) * p.Hv + h) * DV + row,
                                     sm.Dd[t] * rv[e] + ov[e]);
                }
            }
        }
        tc::fence_before_sync();
        ok = !__syncthreads_or(!ok);   // this chunk's tiles and scalars are free
        tc::fence_after_sync();
        if (!ok) break;
        if (tid == 0 && c + 2 < nch) {
            mbar_arrive_expect_tx(&sm.full[buf], kMoBytes + kKeBytes);
            for (int kb = 0; kb < 2; ++kb) {
                tc::tma_load_2d(&sm.Mo[buf][kb * kC * 32], &mo_map, kb * 32, (int)((unit + 2) * kC), &sm.full[buf]);
                tc::tma_load_2d(&sm.Ke[buf][kb * DK * 32], &ke_map, kb * 32, (int)((unit + 2) * DK), &sm.full[buf]);
            }
        }
    }

    // Final state out of tensor memory.
    if (ok) {
        float* dst = p.state_out + (head * DV + row) * DK;
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) {
            float v[32];
            tc::tmem_ld16(lanebase + kColS + 64 * half + 32 * cb, *reinterpret_cast<float(*)[16]>(&v[0]));
            tc::tmem_ld16(lanebase + kColS + 64 * half + 32 * cb + 16, *reinterpret_cast<float(*)[16]>(&v[16]));
#pragma unroll
            for (int q = 0; q < 8; ++q)
                reinterpret_cast<float4*>(dst + 64 * half + 32 * cb)[q] =
                    make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
    } else if (tid == 0) {
        if (p.status_word) atomicOr(p.status_word, kStatusWaitTimeout);
        for (int i = 0; i < 2; ++i) {
            mbar_wait_bounded(&sm.full[i], 0, kMaxPolls);
            mbar_wait_bounded(&sm.full[i], 1, kMaxPolls);
        }
        mbar_wait_bounded(&sm.mma1, 0, kMaxPolls);
        mbar_wait_bounded(&sm.mma2, 0, kMaxPolls);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

template <typename InT, typename OutT>
cudaError_t launch_tc_prefill(const VerifyArgs& a, void* workspace, cudaStream_t stream) {
    const size_t units = (size_t)a.B * a.Hv * n_chunks_of(a.T);
    float* ws_mo = static_cast<float*>(workspace);
    float* ws_ke = ws_mo + units * kMoFloats;
    float* ws_vec = ws_ke + units * kKeFloats;
    static bool configured = false;   // per process; the attributes are per function
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gdn_prefill_prep_kernel<InT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)sizeof(PrepSmem));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gdn_prefill_scan_kernel<InT, OutT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)sizeof(ScanSmem));
        if (e != cudaSuccess) return e;
        configured = true;
    }
    CUtensorMap mo_map, ke_map;
    cudaError_t e = tc::encode_tmap_f32_sw128(&mo_map, ws_mo, units * kC, kC, kC);
    if (e == cudaSuccess) e = tc::encode_tmap_f32_sw128(&ke_map, ws_ke, units * DK, kC, DK);
    if (e != cudaSuccess) return e;
    dim3 pgrid((unsigned)n_chunks_of(a.T), a.Hv, a.B);
    gdn_prefill_prep_kernel<InT><<<pgrid, kThreads, sizeof(PrepSmem), stream>>>(a, ws_mo, ws_ke, ws_vec);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 sgrid(a.Hv, a.B);
    gdn_prefill_scan_kernel<InT, OutT><<<sgrid, kThreads, sizeof(ScanSmem), stream>>>(mo_map, ke_map, a, ws_vec);
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

size_t prefill_workspace_bytes(int B, int T, int Hv, int dk, int dv, int chunk) {
    (void)dk;
    (void)dv;
    (void)chunk;
    const size_t units = (size_t)B * Hv * n_chunks_of(T);
    return units * (kMoFloats + kKeFloats + kVecFloats) * sizeof(float);
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
