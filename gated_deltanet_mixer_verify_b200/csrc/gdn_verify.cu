// gdn_verify.cu -- Gated DeltaNet verify / decode mixer and the two-phase commit, sm_100a.
//
// What is computed (the Gated DeltaNet layer mixer over a speculative verify block;
// source pages "Lithos-metal: Qwen3.8-27B on 40-core M5 Max", table "GDN mixer" and the
// runtime paragraph on recurrent-state commit / rollback, and "Qwen 3.8 27B mac m5: 200
// tok/s, audited", sections on fusing layer mixers and on DSpark verification):
//   S_t = alpha_t S_{t-1} (I - beta_t khat_t khat_t^T) + beta_t v_t khat_t^T,  o_t = S_t qhat_t,
// then the state after the accepted prefix L is written back.
//
// How (B200 design). Rows of S (value index i) evolve independently, so a CTA owns a slice
// of R value rows of one head (the pages' "value-column slice"), loads it from HBM exactly
// once into registers, and writes the committed rows exactly once. The T per-token rank-1
// updates are not applied one by one; with G_t the inclusive cumulative log-decay and
// d_t = exp(G_t), every quantity follows from dots against the block's initial state:
//   p0_t = S_0 khat_t,  r0_t = S_0 qhat_t                      (2T dots per row)
//   A[t][s]  = beta_t exp(G_t - G_s) khat_t.khat_s  (s < t),  Tm = (I + A)^-1
//   x_s      = beta_s (v_s - d_s p0_s),   u = Tm x            (u_t = the rule's write vector)
//   o_t      = d_t r0_t + sum_{s<=t} Mo[t][s] x_s,  Mo = Cq Tm,  Cq[t][s] = exp(G_t-G_s) qhat_t.khat_s
//   S_L      = d_{L-1} S_0 + sum_{s<L} x_s Keff_s,  Keff_s = sum_{s<=t<L} exp(G_{L-1}-G_t) Tm[t][s] khat_t
// The T x T algebra is per head and shared by all rows; per state element the kernel does
// 2T fused multiply-adds for the dots and L+1 for the commit. Decays are only formed as
// exp of a difference of cumulative log-decays (never as a ratio), so strong gates whose
// products underflow stay finite.
//
// Thread mapping: TPR = d_k / 16 lanes share a row; each lane holds 16 columns (4 float4 at
// interleaved chunks c, c+TPR, c+2TPR, c+3TPR, so a warp's global and shared accesses are
// contiguous 128-byte runs) of RPT rows. Partial dots are combined across the TPR lanes
// with a halving butterfly: each exchange step sends half of the live values, so a lane
// issues NV/2 + NV/4 + ... shuffles instead of NV log2(TPR).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kColsPerLane = 16;
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ float ld_in(const void* base, size_t i) {
    return to_f(reinterpret_cast<const T*>(base)[i]);
}

template <typename T>
__device__ __forceinline__ void st_out(void* base, size_t i, float x);
template <>
__device__ __forceinline__ void st_out<float>(void* base, size_t i, float x) {
    reinterpret_cast<float*>(base)[i] = x;
}
template <>
__device__ __forceinline__ void st_out<__nv_bfloat16>(void* base, size_t i, float x) {
    reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(kFull, x, off);
    return x;
}

__device__ __forceinline__ float softplus_f(float x) {
    return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));
}

// Halving butterfly over the lanes of a row group (lane bits below 2*OFF). On return a lane
// whose in-group index is c holds, in v[0..max(CNT/TPR,1)), the fully reduced values whose
// original indices start at c*CNT/TPR (CNT >= TPR) or equal c/(TPR/CNT) (CNT < TPR).
template <int CNT, int OFF>
struct Halve {
    static __device__ __forceinline__ void run(float* v, int lane) {
        if constexpr (OFF == 0) {
            return;
        } else if constexpr (CNT >= 2) {
            constexpr int H = CNT / 2;
            const bool upper = (lane & OFF) != 0;
#pragma unroll
            for (int i = 0; i < H; ++i) {
                const float send = upper ? v[i] : v[i + H];
                const float keep = upper ? v[i + H] : v[i];
                v[i] = keep + __shfl_xor_sync(kFull, send, OFF);
            }
            Halve<H, OFF / 2>::run(v, lane);
        } else {
            v[0] += __shfl_xor_sync(kFull, v[0], OFF);
            Halve<1, OFF / 2>::run(v, lane);
        }
    }
};

__device__ __forceinline__ void fma4(float4& r, float s, const float4& k) {
    r.x = fmaf(s, k.x, r.x);
    r.y = fmaf(s, k.y, r.y);
    r.z = fmaf(s, k.z, r.z);
    r.w = fmaf(s, k.w, r.w);
}

// One CTA: rows [blockIdx.x * R, +R) of value head blockIdx.y of sequence blockIdx.z.
// The T tokens of the sequence are taken in blocks of TM; the state slice stays in registers
// from block to block (prefill), and a single block is the verify / decode case.
template <int DK, int TM, int RPT, typename InT, typename OutT>
__global__ void __launch_bounds__(kThreads, 4) gdn_verify_kernel(const VerifyArgs p) {
    constexpr int TPR = DK / kColsPerLane;   // lanes per row
    constexpr int GROUPS = kThreads / TPR;   // row groups per CTA
    constexpr int R = GROUPS * RPT;          // rows per CTA
    constexpr int NV = RPT * 2 * TM;         // partial dots per lane
    constexpr int LD = DK + 4;               // padded shared row (floats)
    constexpr int NF4 = kColsPerLane / 4;    // float4 chunks per lane and row
    constexpr int PER = NV >= TPR ? NV / TPR : 1;
    constexpr int STRIDE = NV >= TPR ? 1 : TPR / NV;
    static_assert(TPR >= 1 && TPR <= 32 && (TPR & (TPR - 1)) == 0, "d_k / 16 must be a power of two");

    __shared__ __align__(16) float sKQ[2 * TM][LD];   // rows 0..TM-1: khat_t, TM..: qhat_t
    __shared__ __align__(16) float sKeff[TM][LD];
    __shared__ __align__(16) float sP[R][2 * TM];     // reduced dots: p0 then r0
    __shared__ float sV[TM][R];
    __shared__ float sG[TM], sBeta[TM], sD[TM];
    __shared__ float sA[TM][TM], sCq[TM][TM], sTm[TM][TM], sMo[TM][TM], sE[TM][TM];
    __shared__ float sDL;
    __shared__ int sL;

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int row0 = blockIdx.x * R;
    const int T = p.T;                 // tokens of the sequence
    const int dv = p.dv;
    const int g = h / (p.Hv / p.Hk);
    const int grp = tid / TPR;
    const int c = tid % TPR;
    const size_t head = (size_t)b * p.Hv + h;
    const bool multi = T > TM;         // prefill: several blocks, each fully committed

    // 1. Issue the state slice loads first; they stay in flight through the prologue.
    float4 S[RPT][NF4];
    {
        const float* src = p.state_in ? p.state_in + head * (size_t)dv * DK : nullptr;
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {
            const int row = row0 + grp * RPT + rr;
#pragma unroll
            for (int m = 0; m < NF4; ++m) {
                if (src && row < dv)
                    S[rr][m] = __ldcs(reinterpret_cast<const float4*>(src + (size_t)row * DK) + c + TPR * m);
                else
                    S[rr][m] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }

    int L = 0;
    for (int t0 = 0; t0 < T; t0 += TM) {
        const int n = min(TM, T - t0);   // tokens in this block
        if (t0 > 0) __syncthreads();     // the previous block is done with shared memory

        // 2. khat_t, qhat_t of key head g, one warp per vector; zero rows for t >= n.
        for (int nv = warp; nv < 2 * TM; nv += kWarps) {
            const bool isq = nv >= TM;
            const int t = isq ? nv - TM : nv;
            float* dst = sKQ[nv];
            if (t < n) {
                const size_t base = (((size_t)b * T + t0 + t) * p.Hk + g) * DK;
                const void* src = isq ? p.q : p.k;
                constexpr int E = (DK + 31) / 32;
                float x[E];
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int j = lane + 32 * e;
                    x[e] = (j < DK) ? ld_in<InT>(src, base + j) : 0.f;
                    ss = fmaf(x[e], x[e], ss);
                }
                ss = warp_sum(ss);
                const float inv = (isq ? p.scale : 1.f) / sqrtf(ss + p.l2_eps);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int j = lane + 32 * e;
                    if (j < DK) dst[j] = x[e] * inv;
                }
            } else {
                for (int j = lane; j < DK; j += 32) dst[j] = 0.f;
            }
        }

        // 3. Gates and the inclusive prefix sum of log-decays (warp 0, lane t = token t).
        if (warp == 0) {
            float gl = 0.f, be = 0.f;
            if (lane < n) {
                const size_t gi = ((size_t)b * T + t0 + lane) * p.Hv + h;
                gl = -expf(p.A_log[h]) * softplus_f(ld_in<InT>(p.a, gi) + p.dt_bias[h]);
                be = 1.f / (1.f + expf(-ld_in<InT>(p.b, gi)));
            }
            float G = gl;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(kFull, G, off);
                if (lane >= off) G += y;
            }
            if (lane < TM) {
                sG[lane] = G;
                sBeta[lane] = be;
                sD[lane] = (lane < n) ? expf(G) : 0.f;
            }
            if (lane == 0) {
                int Lb;
                if (p.always_commit || multi) {
                    Lb = n;
                } else if (p.accept_len) {
                    Lb = p.accept_len[b];
                    if (Lb < 0 || Lb > T) {
                        if (p.status_word && blockIdx.x == 0 && h == 0) atomicOr(p.status_word, 1);
                        Lb = -1;   // out of range: commit nothing
                    }
                } else {
                    Lb = -2;       // two-phase: the state is not written here
                }
                sL = Lb;
            }
        }

        // v_t for this slice's rows.
        for (int e = tid; e < TM * R; e += kThreads) {
            const int t = e / R, i = e % R;
            const int row = row0 + i;
            sV[t][i] = (t < n && row < dv)
                           ? ld_in<InT>(p.v, (((size_t)b * T + t0 + t) * p.Hv + h) * dv + row)
                           : 0.f;
        }
        __syncthreads();

        // 4. Gram coefficients A (strictly lower) and Cq (lower with diagonal), one warp per entry.
        for (int e = warp; e < 2 * TM * TM; e += kWarps) {
            const int kind = e / (TM * TM);
            const int t = (e % (TM * TM)) / TM;
            const int s = e % TM;
            const bool need = (t < n) && (kind == 0 ? s < t : s <= t);
            float acc = 0.f;
            if (need) {
                const float* x = kind == 0 ? sKQ[t] : sKQ[TM + t];
                const float* y = sKQ[s];
                for (int j = lane; j < DK; j += 32) acc = fmaf(x[j], y[j], acc);
                acc = warp_sum(acc);
            }
            if (lane == 0) {
                const float dec = need ? expf(sG[t] - sG[s]) : 0.f;
                if (kind == 0)
                    sA[t][s] = need ? sBeta[t] * dec * acc : 0.f;
                else
                    sCq[t][s] = need ? dec * acc : 0.f;
            }
        }
        __syncthreads();

        // 5. Tm = (I + A)^-1 by forward substitution, one column per thread.
        if (tid < TM) {
            const int s = tid;
            float col[TM];
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                float x = (t == s) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < t; ++m) x = fmaf(-sA[t][m], col[m], x);
                col[t] = (t >= s) ? x : 0.f;
                sTm[t][s] = col[t];
            }
        }
        __syncthreads();

        // 6. Mo = Cq Tm and the commit coefficients E[t][s] = exp(G_{L-1} - G_t) Tm[t][s], s <= t < L.
        L = sL;
        for (int e = tid; e < TM * TM; e += kThreads) {
            const int t = e / TM, s = e % TM;
            float acc = 0.f;
            for (int m = s; m <= t; ++m) acc = fmaf(sCq[t][m], sTm[m][s], acc);
            sMo[t][s] = (s <= t) ? acc : 0.f;
            sE[t][s] = (L > 0 && t < L && s <= t) ? expf(sG[L - 1] - sG[t]) * sTm[t][s] : 0.f;
        }
        if (tid == 0) sDL = (L > 0) ? sD[L - 1] : 1.f;
        __syncthreads();

        // 7. Keff_s = sum_t E[t][s] khat_t (only when a commit is made).
        if (L > 0) {
            for (int e = tid; e < TM * DK; e += kThreads) {
                const int s = e / DK, j = e % DK;
                float acc = 0.f;
#pragma unroll
                for (int t = 0; t < TM; ++t) acc = fmaf(sE[t][s], sKQ[t][j], acc);
                sKeff[s][j] = acc;
            }
        }

        // 8. Dots of the state rows with all khat_t and qhat_t (this lane's 16 columns).
        float acc[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) acc[i] = 0.f;
#pragma unroll
        for (int m = 0; m < NF4; ++m) {
#pragma unroll
            for (int nv = 0; nv < 2 * TM; ++nv) {
                if ((nv % TM) < n) {
                    const float4 w = *reinterpret_cast<const float4*>(&sKQ[nv][4 * (c + TPR * m)]);
#pragma unroll
                    for (int rr = 0; rr < RPT; ++rr) {
                        float a = acc[rr * 2 * TM + nv];
                        a = fmaf(S[rr][m].x, w.x, a);
                        a = fmaf(S[rr][m].y, w.y, a);
                        a = fmaf(S[rr][m].z, w.z, a);
                        a = fmaf(S[rr][m].w, w.w, a);
                        acc[rr * 2 * TM + nv] = a;
                    }
                }
            }
        }

        // 9. Combine across the row group and park the reduced dots in shared memory.
        Halve<NV, TPR / 2>::run(acc, c);
        if (c % STRIDE == 0) {
            const int base = (NV >= TPR) ? c * PER : c / STRIDE;
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                const int vi = base + e;
                sP[grp * RPT + vi / (2 * TM)][vi % (2 * TM)] = acc[e];
            }
        }
        __syncthreads();

        // 10. Per-row write coefficients x_s = beta_s (v_s - d_s p0_s).
        float xs[RPT][TM];
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {
            const int il = grp * RPT + rr;
#pragma unroll
            for (int s = 0; s < TM; ++s) xs[rr][s] = sBeta[s] * (sV[s][il] - sD[s] * sP[il][s]);
        }

        // 11. Outputs: lane c of the group produces tokens c, c + TPR, ...
        for (int t = c; t < n; t += TPR) {
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) {
                const int il = grp * RPT + rr;
                const int row = row0 + il;
                if (row < dv) {
                    float ov = sD[t] * sP[il][TM + t];
#pragma unroll
                    for (int s = 0; s < TM; ++s)
                        if (s <= t) ov = fmaf(sMo[t][s], xs[rr][s], ov);
                    st_out<OutT>(p.o, (((size_t)b * T + t0 + t) * p.Hv + h) * dv + row, ov);
                }
            }
        }

        // 12. Stash for a later gdn_commit (single-block verify): khat, cumulative log-decay, u = Tm x.
        if (p.stash) {
            float* st = p.stash + head * stash_floats_per_head(T, DK, dv);
            const size_t off_u = (size_t)T * DK + (((size_t)T + 3) & ~size_t(3));
            for (int t = c; t < T; t += TPR) {
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr) {
                    const int row = row0 + grp * RPT + rr;
                    if (row < dv) {
                        float u = 0.f;
#pragma unroll
                        for (int s = 0; s < TM; ++s)
                            if (s <= t) u = fmaf(sTm[t][s], xs[rr][s], u);
                        st[off_u + (size_t)t * dv + row] = u;
                    }
                }
            }
            if (blockIdx.x == 0) {
                for (int e = tid; e < T * DK; e += kThreads) st[e] = sKQ[e / DK][e % DK];
                if (tid < T) st[(size_t)T * DK + tid] = sG[tid];
            }
        }

        // 13. Advance the state in registers: S <- d_{L-1} S + sum_{s<L} x_s Keff_s.
        if (L > 0) {
            const float dl = sDL;
#pragma unroll
            for (int m = 0; m < NF4; ++m) {
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr) {
                    S[rr][m].x *= dl;
                    S[rr][m].y *= dl;
                    S[rr][m].z *= dl;
                    S[rr][m].w *= dl;
                }
#pragma unroll
                for (int s = 0; s < TM; ++s) {
                    if (s < L) {
                        const float4 ke = *reinterpret_cast<const float4*>(&sKeff[s][4 * (c + TPR * m)]);
#pragma unroll
                        for (int rr = 0; rr < RPT; ++rr) fma4(S[rr][m], xs[rr][s], ke);
                    }
                }
            }
        }
    }

    // 14. Write the committed state. Rollback / bad L: the initial state (skipped when in
    // place). Two-phase (L == -2): no state write.
    if (L != -2 && !(L <= 0 && p.state_out == p.state_in)) {
        float* dst = p.state_out + head * (size_t)dv * DK;
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {
            const int row = row0 + grp * RPT + rr;
            if (row < dv) {
#pragma unroll
                for (int m = 0; m < NF4; ++m)
                    __stcs(reinterpret_cast<float4*>(dst + (size_t)row * DK) + c + TPR * m, S[rr][m]);
            }
        }
    }
}

// Second phase: S_L = exp(G_{L-1}) S_0 + sum_{t<L} exp(G_{L-1} - G_t) u_t khat_t^T.
template <int DK, int RPT>
__global__ void __launch_bounds__(kThreads, 4) gdn_commit_kernel(const CommitArgs p) {
    constexpr int TPR = DK / kColsPerLane;
    constexpr int GROUPS = kThreads / TPR;
    constexpr int R = GROUPS * RPT;
    constexpr int NF4 = kColsPerLane / 4;
    constexpr int TMAX = 16;
    __shared__ __align__(16) float sK[TMAX][DK];
    __shared__ float sW[TMAX];
    __shared__ float sDL;
    __shared__ int sL;

    const int tid = threadIdx.x;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int row0 = blockIdx.x * R;
    const int T = p.T;
    const int dv = p.dv;
    const int grp = tid / TPR;
    const int c = tid % TPR;
    const size_t head = (size_t)b * p.Hv + h;
    const float* st = p.stash + head * stash_floats_per_head(T, DK, dv);
    const size_t off_u = (size_t)T * DK + (((size_t)T + 3) & ~size_t(3));

    if (tid == 0) {
        int L = p.accept_len[b];
        if (L < 0 || L > T) {
            if (p.status_word && blockIdx.x == 0 && h == 0) atomicOr(p.status_word, 1);
            L = 0;
        }
        sL = L;
    }
    __syncthreads();
    const int L = sL;
    if (L == 0 && p.state_out == p.state_in) return;   // rollback in place: nothing to write

    if (L > 0) {
        for (int e = tid; e < L * DK; e += kThreads) sK[e / DK][e % DK] = st[e];
        if (tid < L) sW[tid] = expf(st[(size_t)T * DK + L - 1] - st[(size_t)T * DK + tid]);
        if (tid == 0) sDL = expf(st[(size_t)T * DK + L - 1]);
    }
    __syncthreads();

    const float* src = p.state_in + head * (size_t)dv * DK;
    float* dst = p.state_out + head * (size_t)dv * DK;
#pragma unroll
    for (int rr = 0; rr < RPT; ++rr) {
        const int row = row0 + grp * RPT + rr;
        if (row >= dv) continue;
        float4 r[NF4];
#pragma unroll
        for (int m = 0; m < NF4; ++m)
            r[m] = __ldcs(reinterpret_cast<const float4*>(src + (size_t)row * DK) + c + TPR * m);
        if (L > 0) {
            const float dl = sDL;
#pragma unroll
            for (int m = 0; m < NF4; ++m) {
                r[m].x *= dl;
                r[m].y *= dl;
                r[m].z *= dl;
                r[m].w *= dl;
            }
            for (int t = 0; t < L; ++t) {
                const float w = sW[t] * st[off_u + (size_t)t * dv + row];
#pragma unroll
                for (int m = 0; m < NF4; ++m)
                    fma4(r[m], w, *reinterpret_cast<const float4*>(&sK[t][4 * (c + TPR * m)]));
            }
        }
#pragma unroll
        for (int m = 0; m < NF4; ++m)
            __stcs(reinterpret_cast<float4*>(dst + (size_t)row * DK) + c + TPR * m, r[m]);
    }
}

template <int DK, int TM, typename InT, typename OutT>
cudaError_t launch_verify_t(const VerifyArgs& a, cudaStream_t stream) {
    constexpr int RPT = TM >= 16 ? 1 : 2;
    constexpr int R = (kThreads / (DK / kColsPerLane)) * RPT;
    dim3 grid((a.dv + R - 1) / R, a.Hv, a.B);
    gdn_verify_kernel<DK, TM, RPT, InT, OutT><<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

template <int DK, typename InT, typename OutT>
cudaError_t launch_verify_tm(const VerifyArgs& a, cudaStream_t stream) {
    if (a.T <= 1) return launch_verify_t<DK, 1, InT, OutT>(a, stream);
    if (a.T <= 2) return launch_verify_t<DK, 2, InT, OutT>(a, stream);
    if (a.T <= 4) return launch_verify_t<DK, 4, InT, OutT>(a, stream);
    if (a.T <= 8) return launch_verify_t<DK, 8, InT, OutT>(a, stream);
    return launch_verify_t<DK, 16, InT, OutT>(a, stream);
}

template <int DK>
cudaError_t launch_verify_dk(const VerifyArgs& a, cudaStream_t stream) {
    if (a.in_bf16) {
        return a.out_bf16 ? launch_verify_tm<DK, __nv_bfloat16, __nv_bfloat16>(a, stream)
                          : launch_verify_tm<DK, __nv_bfloat16, float>(a, stream);
    }
    return a.out_bf16 ? launch_verify_tm<DK, float, __nv_bfloat16>(a, stream)
                      : launch_verify_tm<DK, float, float>(a, stream);
}

template <int DK>
cudaError_t launch_commit_dk(const CommitArgs& a, cudaStream_t stream) {
    constexpr int RPT = 2;
    constexpr int R = (kThreads / (DK / kColsPerLane)) * RPT;
    dim3 grid((a.dv + R - 1) / R, a.Hv, a.B);
    gdn_commit_kernel<DK, RPT><<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

thread_local const char* g_last_verify_kernel = "";

const char* last_verify_kernel() { return g_last_verify_kernel; }

cudaError_t launch_verify(const VerifyArgs& a, cudaStream_t stream) {
    int nsm = 0;
    cudaError_t e = current_sm_count(&nsm);
    if (e != cudaSuccess) return e;
    if (pipe_kernel_applies(a, nsm)) {
        g_last_verify_kernel = "gdn_verify_pipe_kernel";
        return launch_verify_pipe(a, stream);
    }
    if (tc_kernel_applies(a, nsm)) {
        g_last_verify_kernel = "gdn_verify_tc_kernel";
        return launch_verify_tc(a, stream);   // fuses the gated norm
    }
    // Other kernels: the mixer writes o, then the gated norm runs over o in place.
    VerifyArgs m = a;
    m.norm_z = nullptr;
    if (rec_kernel_applies(m, nsm)) {
        g_last_verify_kernel = "gdn_verify_rec_kernel";
        e = launch_verify_rec(m, stream);
    } else if (head_kernel_applies(m)) {
        g_last_verify_kernel = "gdn_verify_head_kernel";
        e = launch_verify_head(m, stream);
    } else {
        g_last_verify_kernel = "gdn_verify_kernel";
        switch (m.dk) {
            case 16: e = launch_verify_dk<16>(m, stream); break;
            case 32: e = launch_verify_dk<32>(m, stream); break;
            case 64: e = launch_verify_dk<64>(m, stream); break;
            case 128: e = launch_verify_dk<128>(m, stream); break;
            default: return cudaErrorInvalidValue;
        }
    }
    if (e != cudaSuccess || !a.norm_z) return e;
    NormArgs n;
    n.x = a.o;
    n.z = a.norm_z;
    n.w = a.norm_w;
    n.y = a.o;
    n.rows = (int64_t)a.B * a.T * a.Hv;
    n.d = a.dv;
    n.eps = a.norm_eps;
    n.x_bf16 = a.out_bf16 != 0;
    n.z_bf16 = a.in_bf16 != 0;
    n.y_bf16 = a.out_bf16 != 0;
    return launch_gated_rmsnorm(n, stream);
}

cudaError_t launch_commit(const CommitArgs& a, cudaStream_t stream) {
    switch (a.dk) {
        case 16: return launch_commit_dk<16>(a, stream);
        case 32: return launch_commit_dk<32>(a, stream);
        case 64: return launch_commit_dk<64>(a, stream);
        case 128: return launch_commit_dk<128>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gdn
