// gdn_verify_rec.cu -- latency form of the verify / decode mixer for small batches (fewer
// (sequence, value head) pairs than SMs), d_k = 128, T <= 16, with the commit fused at device
// accept counts (or every token committed, for decode).
//
// With one sequence a layer has 48 heads: the work is a few microseconds of dependent steps,
// not bandwidth. This kernel runs the rule literally, token by token, on rows of a head's
// state held in registers, so that nothing waits on a block barrier once the block's
// normalised keys, queries and gates are known:
//   p_t = S_{t-1} khat_t,  r_t = S_{t-1} qhat_t          (8 lanes per row, shuffles)
//   u_t = beta_t (v_t - alpha_t p_t)
//   o_t = alpha_t r_t + u_t (khat_t . qhat_t)           (= S_t qhat_t)
//   S_t = alpha_t S_{t-1} + u_t khat_t^T                (= alpha_t S_{t-1}(I - beta_t khat khat^T) + beta_t v khat^T)
// and S_L leaves for state_out as soon as token L - 1 is done (L = 0: nothing, or S_0 when
// written out of place). One CTA (128 threads) per (sequence, value head, 16 R rows); a thread
// holds columns 32 m + 4 j .. +3 (m = 0..3, j = its lane in the row's group of 8) of R rows,
// rg + 16 i, so each normalised key and query it reads from shared memory serves R rows (with
// one row per thread the token loop was bound by those reads) and a row's stores are 128-byte
// runs. The q/k normalisation is computed by every CTA of a head.
//
// Programmatic dependent launch (VerifyArgs::pdl): the state rows are loaded into registers
// and the block's q, k, v rows and gate inputs prefetched into L2 before griddepcontrol.wait;
// every other read, and every write, comes after it (a prefetch hands the thread no data, and
// the L2 is coherent, so a write by the kernel before still reaches the loads after the wait).
// Without the gate prefetch the gates came from HBM after the wait and were the last input to
// arrive. The next kernel is released once this block has staged its inputs (after the block
// barrier): released at entry, the next layer's blocks sat on their SMs through this layer's
// input loads and made the layer slower.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.cuh"

namespace gdn {
namespace {
using namespace dev;

constexpr int kThreads = 128;
constexpr int DK = 128;
constexpr int kLanes = 8;                  // lanes per row group
constexpr int kGroups = kThreads / kLanes;
constexpr int kR = 2;                      // rows per thread (1 and 4 measured slower)
constexpr int kRowsCta = kGroups * kR;

// Four consecutive input elements from element i (a multiple of 4) of a 16-byte aligned array:
// one 8-byte load for bf16, one 16-byte load for fp32.
template <typename T>
__device__ __forceinline__ void ld4_in(const void* base, size_t i, float* x);
template <>
__device__ __forceinline__ void ld4_in<float>(const void* base, size_t i, float* x) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i));
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}
template <>
__device__ __forceinline__ void ld4_in<__nv_bfloat16>(const void* base, size_t i, float* x) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(base) + i));
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xffff0000u);
}

template <int TM>
struct RecSmem {
    alignas(16) float KQ[2 * TM][DK];   // khat_t (rows < TM), qhat_t (rows >= TM), normalised
    float alpha[TM], beta[TM], kq[TM];
    int L;
};

template <int TM, typename InT, typename OutT>
__global__ void __launch_bounds__(kThreads) gdn_verify_rec_kernel(const VerifyArgs p) {
    constexpr int NO = TM / kLanes;           // outputs a lane stores per row
    __shared__ RecSmem<TM> sm;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int T = p.T;
    const int dv = p.dv;
    const int slices = dv / kRowsCta;
    const int item = blockIdx.x;
    const int sl = item % slices;
    const int h = (item / slices) % p.Hv;
    const int b = item / slices / p.Hv;
    const int g = h / (p.Hv / p.Hk);
    const int rg = tid / kLanes;              // row group: rows rg + 16 i of the slice
    const int j = tid % kLanes;               // lane within the row group
    const size_t row0 = ((size_t)b * p.Hv + h) * dv + (size_t)sl * kRowsCta + rg;   // state row of row i = 0

    // 1. This thread's rows of state into registers (never written by the kernel before).
    float4 S[kR][4];
#pragma unroll
    for (int i = 0; i < kR; ++i) {
        const float4* src = reinterpret_cast<const float4*>(p.state_in + (row0 + kGroups * i) * DK);
#pragma unroll
        for (int m = 0; m < 4; ++m) S[i][m] = src[8 * m + j];
    }
    if (p.pdl && sl == 0) {   // the block's q, k, v rows and gate inputs into L2 (once per head)
        const size_t el = p.in_bf16 ? 2 : 4;
        if (tid < 3 * T) {
            const int t = tid / 3, which = tid % 3;
            const char* base = static_cast<const char*>(which == 0 ? p.q : which == 1 ? p.k : p.v);
            const size_t off = which < 2 ? (((size_t)b * T + t) * p.Hk + g) * DK : (((size_t)b * T + t) * p.Hv + h) * dv;
            bulk_prefetch_l2(base + off * el, (uint32_t)((which < 2 ? DK : dv) * el));   // rows of 16-byte multiples
        } else if (warp == 3) {               // 3 T <= 48 < 96
            if (lane < T) {
                const size_t gi = (((size_t)b * T + lane) * p.Hv + h) * el;
                prefetch_l2_line(static_cast<const char*>(p.a) + gi);
                prefetch_l2_line(static_cast<const char*>(p.b) + gi);
            } else if (lane == 31) {
                prefetch_l2_line(p.A_log + h);
                prefetch_l2_line(p.dt_bias + h);
            }
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // 2. Token t's k and q rows for 16 lanes (tid / 16 = t mod 8, 8 columns each: 64 m + 4 c + e),
    // v_t of this thread's rows, and the gates (warp 0, lane t = token t); every load first.
    const int c16 = tid & 15;
    const int tt = tid >> 4;
    float kx[TM / 8][8], qx[TM / 8][8];
#pragma unroll
    for (int e2 = 0; e2 < TM / 8; ++e2) {
        const int t = tt + 8 * e2;
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const size_t base = (((size_t)b * T + t) * p.Hk + g) * DK + 64 * m + 4 * c16;
            if (t < T) {
                ld4_in<InT>(p.k, base, &kx[e2][4 * m]);
                ld4_in<InT>(p.q, base, &qx[e2][4 * m]);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) kx[e2][4 * m + e] = qx[e2][4 * m + e] = 0.f;
            }
        }
    }
    const size_t vrow0 = (size_t)sl * kRowsCta + rg;    // value row of row i = 0 within the head
    float vr[kR][TM];
#pragma unroll
    for (int i = 0; i < kR; ++i)
#pragma unroll
        for (int t = 0; t < TM; ++t)
            vr[i][t] = (t < T) ? ld_in<InT>(p.v, (((size_t)b * T + t) * p.Hv + h) * dv + vrow0 + kGroups * i) : 0.f;
    float a_in = 0.f, b_in = 0.f, alog = 0.f, dtb = 0.f;
    int L_in = 0;
    if (warp == 0) {
        if (lane < T) {
            const size_t gi = ((size_t)b * T + lane) * p.Hv + h;
            a_in = ld_in<InT>(p.a, gi);
            b_in = ld_in<InT>(p.b, gi);
        }
        alog = p.A_log[h];
        dtb = p.dt_bias[h];
        if (!p.always_commit) L_in = p.accept_len[b];
    }
    // Sums of k^2, q^2 and k.q over the 128 columns (the token's 16 lanes), the normalised rows.
#pragma unroll
    for (int e2 = 0; e2 < TM / 8; ++e2) {
        const int t = tt + 8 * e2;
        float sk = 0.f, sq = 0.f, skq = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            sk = fmaf(kx[e2][e], kx[e2][e], sk);
            sq = fmaf(qx[e2][e], qx[e2][e], sq);
            skq = fmaf(kx[e2][e], qx[e2][e], skq);
        }
        sk = group_sum<16>(sk);
        sq = group_sum<16>(sq);
        skq = group_sum<16>(skq);
        const bool live = t < T;
        const float ik = live ? rsqrtf(sk + p.l2_eps) : 0.f;
        const float iq = live ? p.scale * rsqrtf(sq + p.l2_eps) : 0.f;
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            *reinterpret_cast<float4*>(&sm.KQ[t][64 * m + 4 * c16]) =
                make_float4(kx[e2][4 * m] * ik, kx[e2][4 * m + 1] * ik, kx[e2][4 * m + 2] * ik, kx[e2][4 * m + 3] * ik);
            *reinterpret_cast<float4*>(&sm.KQ[TM + t][64 * m + 4 * c16]) =
                make_float4(qx[e2][4 * m] * iq, qx[e2][4 * m + 1] * iq, qx[e2][4 * m + 2] * iq, qx[e2][4 * m + 3] * iq);
        }
        if (c16 == 0) sm.kq[t] = skq * ik * iq;
    }
    if (warp == 0) {
        float gl = 0.f, be = 0.f;
        if (lane < T) {
            gl = -expf(alog) * softplus_f(a_in + dtb);
            be = 1.f / (1.f + expf(-b_in));
        }
        if (lane < TM) {
            sm.alpha[lane] = (lane < T) ? expf(gl) : 1.f;
            sm.beta[lane] = be;
        }
        if (lane == 0) {
            int L;
            if (p.always_commit) {
                L = T;
            } else {
                L = L_in;
                if (L < 0 || L > T) {
                    if (p.status_word && h == 0 && sl == 0) atomicOr(p.status_word, kStatusBadAccept);
                    L = -1;
                }
            }
            sm.L = L;
        }
    }
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // 3. The recurrence over the block, committing S_L when token L - 1 is done.
    const int L = sm.L;
    const bool in_place = p.state_out == p.state_in;
    if (L <= 0 && !in_place) {   // rollback / bad count out of place: S_0 as it was
#pragma unroll
        for (int i = 0; i < kR; ++i) {
            float4* dst = reinterpret_cast<float4*>(p.state_out + (row0 + kGroups * i) * DK);
#pragma unroll
            for (int m = 0; m < 4; ++m) __stcs(dst + 8 * m + j, S[i][m]);
        }
    }
    float o_keep[kR][NO > 0 ? NO : 1];
#pragma unroll
    for (int i = 0; i < kR; ++i)
#pragma unroll
        for (int e = 0; e < (NO > 0 ? NO : 1); ++e) o_keep[i][e] = 0.f;
#pragma unroll
    for (int t = 0; t < TM; ++t) {
        if (t < T) {
            float4 kk[4], qq[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                kk[m] = *reinterpret_cast<const float4*>(&sm.KQ[t][32 * m + 4 * j]);
                qq[m] = *reinterpret_cast<const float4*>(&sm.KQ[TM + t][32 * m + 4 * j]);
            }
            float pv[kR], rv[kR];
#pragma unroll
            for (int i = 0; i < kR; ++i) {
                float2 pa = make_float2(0.f, 0.f), ra = make_float2(0.f, 0.f);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    pa = __ffma2_rn(make_float2(S[i][m].x, S[i][m].y), make_float2(kk[m].x, kk[m].y), pa);
                    pa = __ffma2_rn(make_float2(S[i][m].z, S[i][m].w), make_float2(kk[m].z, kk[m].w), pa);
                    ra = __ffma2_rn(make_float2(S[i][m].x, S[i][m].y), make_float2(qq[m].x, qq[m].y), ra);
                    ra = __ffma2_rn(make_float2(S[i][m].z, S[i][m].w), make_float2(qq[m].z, qq[m].w), ra);
                }
                pv[i] = pa.x + pa.y;
                rv[i] = ra.x + ra.y;
            }
#pragma unroll
            for (int off = kLanes / 2; off >= 1; off >>= 1)
#pragma unroll
                for (int i = 0; i < kR; ++i) {
                    pv[i] += __shfl_xor_sync(kFull, pv[i], off);
                    rv[i] += __shfl_xor_sync(kFull, rv[i], off);
                }
            const float al = sm.alpha[t], be = sm.beta[t], kqt = sm.kq[t];
            const float2 a2 = make_float2(al, al);
#pragma unroll
            for (int i = 0; i < kR; ++i) {
                const float u = be * (vr[i][t] - al * pv[i]);
                const float ov = fmaf(al, rv[i], u * kqt);
                if (j == (t % kLanes)) o_keep[i][t / kLanes] = ov;
                const float2 u2 = make_float2(u, u);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float2 lo = __ffma2_rn(u2, make_float2(kk[m].x, kk[m].y), __fmul2_rn(a2, make_float2(S[i][m].x, S[i][m].y)));
                    const float2 hi = __ffma2_rn(u2, make_float2(kk[m].z, kk[m].w), __fmul2_rn(a2, make_float2(S[i][m].z, S[i][m].w)));
                    S[i][m] = make_float4(lo.x, lo.y, hi.x, hi.y);
                }
            }
            if (t + 1 == L) {
#pragma unroll
                for (int i = 0; i < kR; ++i) {
                    float4* dst = reinterpret_cast<float4*>(p.state_out + (row0 + kGroups * i) * DK);
#pragma unroll
                    for (int m = 0; m < 4; ++m) __stcs(dst + 8 * m + j, S[i][m]);
                }
            }
        }
    }
    // Outputs: lane j holds o_j (and o_{j+8}) of each of its rows.
    OutT* op = reinterpret_cast<OutT*>(p.o);
#pragma unroll
    for (int i = 0; i < kR; ++i)
#pragma unroll
        for (int e = 0; e < (NO > 0 ? NO : 1); ++e) {
            const int t = j + kLanes * e;
            if (t < T) st_out<OutT>(op, (((size_t)b * T + t) * p.Hv + h) * dv + vrow0 + kGroups * i, o_keep[i][e]);
        }
}

template <int TM, typename InT, typename OutT>
cudaError_t launch_rec_t(const VerifyArgs& a, cudaStream_t stream) {
    const int grid = a.B * a.Hv * (a.dv / kRowsCta);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gdn_verify_rec_kernel<TM, InT, OutT>, a);
}

template <typename InT, typename OutT>
cudaError_t launch_rec_tm(const VerifyArgs& a, cudaStream_t stream) {
    if (a.T <= 8) return launch_rec_t<8, InT, OutT>(a, stream);
    return launch_rec_t<16, InT, OutT>(a, stream);
}

}  // namespace

bool rec_kernel_applies(const VerifyArgs& a, int num_sms) {
    return a.dk == DK && a.dv % kRowsCta == 0 && a.T >= 1 && a.T <= 16 && (long long)a.B * a.Hv < num_sms &&
           (a.accept_len || a.always_commit) && a.state_out && !a.stash && !a.prev_stash;
}

cudaError_t launch_verify_rec(const VerifyArgs& a, cudaStream_t stream) {
    if (a.in_bf16)
        return a.out_bf16 ? launch_rec_tm<__nv_bfloat16, __nv_bfloat16>(a, stream)
                          : launch_rec_tm<__nv_bfloat16, float>(a, stream);
    return a.out_bf16 ? launch_rec_tm<float, __nv_bfloat16>(a, stream) : launch_rec_tm<float, float>(a, stream);
}

}  // namespace gdn
