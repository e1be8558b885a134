// gdn_verify_head.cu -- one CTA per (sequence, value head) form of the verify / decode mixer
// for d_k = 128, d_v <= 128 (the model-scale shapes).
//
// The math is the block form described in gdn_verify.cu (dots against the block's initial
// state, a T x T unit-triangular solve for the write vectors, folded commit keys). What this
// kernel changes is the schedule:
//   - the head's whole 64 KB fp32 state is requested at once by four bulk asynchronous copies
//     (cp.async.bulk, one mbarrier per 32-row quarter) issued before anything else, so the HBM
//     reads are in flight while the per-head algebra runs;
//   - that algebra (q/k L2 norm, gates, the Gram matrices, (I + A)^-1, the output and commit
//     coefficients) is computed once per head by all 256 threads in parallel instead of once
//     per 32-row slice;
//   - the rows are then streamed in passes of 64: dots from shared memory, a halving
//     butterfly across the 8 lanes of a row, outputs, and the committed rows written with
//     streaming stores.
// Every mbarrier wait is bounded; a wait that runs out sets GDN_STATUS_WAIT_TIMEOUT in the
// status word, suppresses this CTA's global writes, waits (bounded) for its copies and ends.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.cuh"

namespace gdn {
namespace {
using namespace dev;

constexpr int kThreads = 256;
constexpr int DK = 128;
constexpr int TPR = 8;                 // lanes per row in the streaming passes (16 columns each)
constexpr int GROUPS = kThreads / TPR; // 32 row groups
constexpr int LD = DK + 4;             // padded row of the key / query tiles
constexpr int kMaxRows = 128;
constexpr int kQuarter = 32;           // rows per bulk copy / mbarrier
constexpr uint32_t kMaxPolls = 1u << 24;

template <int TM, int RPT>
struct __align__(16) HeadSmem {
    float S[kMaxRows][DK];             // the head's state, filled by bulk copies
    float KQ[2 * TM][LD];              // khat_t (rows < TM), qhat_t (rows >= TM)
    float Keff[TM][LD];
    float V[TM][kMaxRows];
    float P[GROUPS * RPT][2 * TM + 1]; // reduced dots of the current pass (padded row)
    float Gram[2 * TM][TM];            // khat_t.khat_s, then qhat_t.khat_s
    float G[TM], Beta[TM], D[TM];
    float A[TM][TM], Cq[TM][TM], Tm[TM][TM], Mo[TM][TM], E[TM][TM];
    float DL;
    int L;
    int refilled;                      // quarters of the next item already requested
    uint64_t bar[kMaxRows / kQuarter];
};

template <int TM, int RPT, typename InT, typename OutT>
__global__ void __launch_bounds__(kThreads, 2) gdn_verify_head_kernel(const VerifyArgs p) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    HeadSmem<TM, RPT>& sm = *reinterpret_cast<HeadSmem<TM, RPT>*>(smem_raw);
    constexpr int NVH = RPT * TM;                          // dots per lane per half
    constexpr int PER = NVH >= TPR ? NVH / TPR : 1;
    constexpr int STRIDE = NVH >= TPR ? 1 : TPR / NVH;
    constexpr int GPER = TM >= 16 ? TM / 16 : 1;        // Gram values per lane after reduction
    constexpr int GSTRIDE = TM >= 16 ? 1 : 16 / TM;

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int T = p.T;
    const int dv = p.dv;
    const int nsplit = p.row_split;                 // CTAs (items) per head
    const int n_items = p.B * p.Hv * nsplit;
    const int rows_item = dv / nsplit;               // a multiple of 32 when nsplit > 1
    const int nq = (rows_item + kQuarter - 1) / kQuarter;

    // Issue quarter copies [q0, q1) of item `it` into the stages (thread 0 only).
    auto request_quarters = [&](int it, int q0, int q1) {
        const float* src = p.state_in + ((size_t)(it / nsplit) * dv + (size_t)(it % nsplit) * rows_item) * DK;
        for (int q = q0; q < q1 && q < nq; ++q) {
            const int rows = min(kQuarter, rows_item - kQuarter * q);
            const uint32_t bytes = (uint32_t)rows * DK * sizeof(float);
            mbar_arrive_expect_tx(&sm.bar[q], bytes);
            bulk_g2s(&sm.S[kQuarter * q][0], src + (size_t)kQuarter * q * DK, bytes, &sm.bar[q]);
        }
    };

    // 0. Request the first head's state.
    if (tid == 0) {
#pragma unroll
        for (int q = 0; q < kMaxRows / kQuarter; ++q) mbar_init(&sm.bar[q], 1);
        fence_barrier_init();
        if ((int)blockIdx.x < n_items) request_quarters(blockIdx.x, 0, nq);
    }
    // Programmatic dependent launch (a no-op in plain stream order): the next kernel on the
    // stream may start now; this one brings its first item's q, k, v rows and gate inputs into
    // L2 (the L2 is coherent, so a later write by the kernel before it is still seen), and waits
    // for that kernel to complete before it reads any other input or writes anything.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (p.pdl && (int)blockIdx.x < n_items && tid < 3 * T) {
        const int it = blockIdx.x;
        const int hh = (it / nsplit) % p.Hv, bb = it / nsplit / p.Hv, gg = hh / (p.Hv / p.Hk);
        const int t = tid / 3, which = tid % 3;
        const size_t el = p.in_bf16 ? 2 : 4;
        const char* base = static_cast<const char*>(which == 0 ? p.q : which == 1 ? p.k : p.v);
        const size_t off = which < 2 ? (((size_t)bb * T + t) * p.Hk + gg) * DK : (((size_t)bb * T + t) * p.Hv + hh) * dv;
        const uint32_t bytes = (uint32_t)((which < 2 ? DK : dv) * el) & ~15u;
        const char* src = base + off * el;
        // A bulk prefetch needs a 16-byte aligned start (v rows of odd d_v may not have one).
        if (bytes && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) bulk_prefetch_l2(src, bytes);
    }
    if (p.pdl && (int)blockIdx.x < n_items && tid >= kThreads - 32) {   // and its gate inputs
        const int it = blockIdx.x;
        const int hh = (it / nsplit) % p.Hv, bb = it / nsplit / p.Hv;
        const int ln = tid - (kThreads - 32);
        const size_t el = p.in_bf16 ? 2 : 4;
        for (int t = ln; t < T; t += 32) {
            const size_t gi = (((size_t)bb * T + t) * p.Hv + hh) * el;
            prefetch_l2_line(static_cast<const char*>(p.a) + gi);
            prefetch_l2_line(static_cast<const char*>(p.b) + gi);
        }
        if (ln == 0) {
            prefetch_l2_line(p.A_log + hh);
            prefetch_l2_line(p.dt_bias + hh);
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");

    bool ok = true;
    uint32_t parity = 0;   // phase of every stage's barrier for the current item
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, parity ^= 1u) {
    if (tid == 0) sm.refilled = 0;
    const int sp = item % nsplit;
    const int h = (item / nsplit) % p.Hv;
    const int b = item / nsplit / p.Hv;
    const int g = h / (p.Hv / p.Hk);
    const size_t head = (size_t)b * p.Hv + h;
    const int row_base = sp * rows_item;             // first state row of this item
    const int next = item + gridDim.x;

    // 1a. khat_t and qhat_t: 16 lanes per vector, 8 columns per lane.
    {
        const int c16 = tid & 15;
        for (int base = 0; base < 2 * TM; base += kThreads / 16) {
            const int n = base + (tid >> 4);
            const bool isq = n >= TM;
            const int t = isq ? n - TM : n;
            const bool live = n < 2 * TM && t < T;
            float x[8];
            if (live) {
                ld8<InT>(isq ? p.q : p.k, (((size_t)b * T + t) * p.Hk + g) * DK + 8 * c16, x);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = 0.f;
            }
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
            ss = group_sum<16>(ss);
            const float inv = live ? (isq ? p.scale : 1.f) / sqrtf(ss + p.l2_eps) : 0.f;
            if (n < 2 * TM) {
                float4* d = reinterpret_cast<float4*>(&sm.KQ[n][8 * c16]);
                d[0] = make_float4(x[0] * inv, x[1] * inv, x[2] * inv, x[3] * inv);
                d[1] = make_float4(x[4] * inv, x[5] * inv, x[6] * inv, x[7] * inv);
            }
        }
    }

    // 1b. Gates and the inclusive prefix sum of log-decays (warp 0, lane t = token t).
    if (warp == 0) {
        float gl = 0.f, be = 0.f;
        if (lane < T) {
            const size_t gi = ((size_t)b * T + lane) * p.Hv + h;
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
            sm.G[lane] = G;
            sm.Beta[lane] = be;
            sm.D[lane] = (lane < T) ? expf(G) : 0.f;
        }
        if (lane == 0) {
            int L;
            if (p.always_commit) {
                L = T;
            } else if (p.accept_len) {
                L = p.accept_len[b];
                if (L < 0 || L > T) {
                    if (p.status_word && h == 0 && sp == 0) atomicOr(p.status_word, kStatusBadAccept);
                    L = -1;
                }
            } else {
                L = -2;
            }
            sm.L = L;
        }
    }

    // 1c. v_t for every row of the head.
    for (int e = tid; e < TM * kMaxRows; e += kThreads) {
        const int t = e / kMaxRows, i = e % kMaxRows;
        sm.V[t][i] = (t < T && i < rows_item)
                         ? ld_in<InT>(p.v, (((size_t)b * T + t) * p.Hv + h) * dv + row_base + i)
                         : 0.f;
    }
    __syncthreads();

    // 1d. Gram rows: lane group of 16 per row n of [K; Q], partial dots over 8 columns.
    {
        const int c16 = tid & 15;
        for (int base = 0; base < 2 * TM; base += kThreads / 16) {
            const int n = base + (tid >> 4);
            const bool live = n < 2 * TM;
            float part[TM];
            const float4* xr = reinterpret_cast<const float4*>(&sm.KQ[live ? n : 0][8 * c16]);
            const float4 x0 = xr[0], x1 = xr[1];
#pragma unroll
            for (int s = 0; s < TM; ++s) {
                const float4* yr = reinterpret_cast<const float4*>(&sm.KQ[s][8 * c16]);
                const float4 y0 = yr[0], y1 = yr[1];
                float d = x0.x * y0.x;
                d = fmaf(x0.y, y0.y, d);
                d = fmaf(x0.z, y0.z, d);
                d = fmaf(x0.w, y0.w, d);
                d = fmaf(x1.x, y1.x, d);
                d = fmaf(x1.y, y1.y, d);
                d = fmaf(x1.z, y1.z, d);
                d = fmaf(x1.w, y1.w, d);
                part[s] = d;
            }
            Halve<TM, 8>::run(part, c16);
            if (live && c16 % GSTRIDE == 0) {
                const int i0 = TM >= 16 ? c16 * GPER : c16 / GSTRIDE;
#pragma unroll
                for (int e = 0; e < GPER; ++e) sm.Gram[n][i0 + e] = part[e];
            }
        }
    }
    __syncthreads();

    // 1e. Decayed coefficient matrices A (strictly lower) and Cq (lower with diagonal).
    for (int e = tid; e < TM * TM; e += kThreads) {
        const int t = e / TM, s = e % TM;
        const bool inq = t < T && s <= t;
        const float dec = inq ? expf(sm.G[t] - sm.G[s]) : 0.f;
        sm.A[t][s] = (inq && s < t) ? sm.Beta[t] * dec * sm.Gram[t][s] : 0.f;
        sm.Cq[t][s] = inq ? dec * sm.Gram[TM + t][s] : 0.f;
    }
    __syncthreads();

    // 1f. Tm = (I + A)^-1, one column per thread.
    if (tid < TM) {
        const int s = tid;
        float col[TM];
#pragma unroll
        for (int t = 0; t < TM; ++t) {
            float x = (t == s) ? 1.f : 0.f;
#pragma unroll
            for (int m = 0; m < t; ++m) x = fmaf(-sm.A[t][m], col[m], x);
            col[t] = (t >= s) ? x : 0.f;
            sm.Tm[t][s] = col[t];
        }
    }
    __syncthreads();

    // 1g. Mo = Cq Tm and the commit coefficients E[t][s] = exp(G_{L-1} - G_t) Tm[t][s].
    const int L = sm.L;
    for (int e = tid; e < TM * TM; e += kThreads) {
        const int t = e / TM, s = e % TM;
        float acc = 0.f;
        for (int m = s; m <= t; ++m) acc = fmaf(sm.Cq[t][m], sm.Tm[m][s], acc);
        sm.Mo[t][s] = (s <= t) ? acc : 0.f;
        sm.E[t][s] = (L > 0 && t < L && s <= t) ? expf(sm.G[L - 1] - sm.G[t]) * sm.Tm[t][s] : 0.f;
    }
    if (tid == 0) sm.DL = (L > 0) ? sm.D[L - 1] : 1.f;
    __syncthreads();

    // 1h. Keff_s = sum_t E[t][s] khat_t.
    if (L > 0) {
        for (int e = tid; e < TM * DK; e += kThreads) {
            const int s = e / DK, j = e % DK;
            float acc = 0.f;
#pragma unroll
            for (int t = 0; t < TM; ++t) acc = fmaf(sm.E[t][s], sm.KQ[t][j], acc);
            sm.Keff[s][j] = acc;
        }
    }
    __syncthreads();

    // 2. Stream the rows in passes of GROUPS * RPT.
    const int grp = tid / TPR;
    const int c = tid % TPR;
    const float dl = sm.DL;
    const bool write_state = (L != -2) && !(L <= 0 && p.state_out == p.state_in);
    float* dst = write_state ? p.state_out + head * (size_t)dv * DK : nullptr;
    for (int r0 = 0; r0 < rows_item; r0 += GROUPS * RPT) {
        const int q0 = r0 / kQuarter;
        const int q1 = min(nq, (r0 + GROUPS * RPT + kQuarter - 1) / kQuarter);
        for (int q = q0; q < q1; ++q) {
            if (!mbar_wait_bounded(&sm.bar[q], parity, kMaxPolls)) {
                if (ok && p.status_word) atomicOr(p.status_word, kStatusWaitTimeout);
                ok = false;
            }
        }

        float4 S[RPT][4];
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {
            const int lr = r0 + grp * RPT + rr;     // row within this item
#pragma unroll
            for (int m = 0; m < 4; ++m)
                S[rr][m] = lr < rows_item ? *reinterpret_cast<const float4*>(&sm.S[lr][4 * (c + TPR * m)])
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
        }

        // Dots with khat (half 0) then qhat (half 1): packed fp32 FMAs over column pairs,
        // then a halving butterfly over the row's 8 lanes, parked in P.
        __syncwarp();   // this group's previous pass has finished reading P
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float2 a2[RPT][TM];
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
                for (int n = 0; n < TM; ++n) a2[rr][n] = make_float2(0.f, 0.f);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
#pragma unroll
                for (int n = 0; n < TM; ++n) {
                    if (n < T) {
                        const float4 w = *reinterpret_cast<const float4*>(&sm.KQ[half * TM + n][4 * (c + TPR * m)]);
                        const float2 wlo = make_float2(w.x, w.y), whi = make_float2(w.z, w.w);
#pragma unroll
                        for (int rr = 0; rr < RPT; ++rr) {
                            a2[rr][n] = __ffma2_rn(make_float2(S[rr][m].x, S[rr][m].y), wlo, a2[rr][n]);
                            a2[rr][n] = __ffma2_rn(make_float2(S[rr][m].z, S[rr][m].w), whi, a2[rr][n]);
                        }
                    }
                }
            }
            float acc[NVH];
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
                for (int n = 0; n < TM; ++n) acc[rr * TM + n] = a2[rr][n].x + a2[rr][n].y;
            Halve<NVH, TPR / 2>::run(acc, c);
            if (c % STRIDE == 0) {
                const int base = (NVH >= TPR) ? c * PER : c / STRIDE;
#pragma unroll
                for (int e = 0; e < PER; ++e) {
                    const int vi = base + e;
                    sm.P[grp * RPT + vi / TM][half * TM + vi % TM] = acc[e];
                }
            }
        }
        __syncwarp();

        // x_s = beta_s (v_s - d_s p0_s) for this lane's rows.
        float xs[RPT][TM];
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {
            const int il = grp * RPT + rr;
            const int lr = min(r0 + il, kMaxRows - 1);
#pragma unroll
            for (int s = 0; s < TM; ++s) xs[rr][s] = sm.Beta[s] * (sm.V[s][lr] - sm.D[s] * sm.P[il][s]);
        }

        // Outputs: lane c produces tokens c, c + TPR, ...
        for (int t = c; t < T; t += TPR) {
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) {
                const int il = grp * RPT + rr;
                const int row = row_base + r0 + il;
                if (ok && r0 + il < rows_item) {
                    float ov = sm.D[t] * sm.P[il][TM + t];
#pragma unroll
                    for (int s = 0; s < TM; ++s)
                        if (s <= t) ov = fmaf(sm.Mo[t][s], xs[rr][s], ov);
                    st_out<OutT>(p.o, (((size_t)b * T + t) * p.Hv + h) * dv + row, ov);
                }
            }
        }

        // Stash for a later gdn_commit: u = Tm x (rows), and khat / G once per head.
        if (p.stash && ok) {
            float* st = p.stash + head * stash_floats_per_head(T, DK, dv);
            const size_t off_u = (size_t)T * DK + (((size_t)T + 3) & ~size_t(3));
            for (int t = c; t < T; t += TPR) {
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr) {
                    const int lr = r0 + grp * RPT + rr;
                    const int row = row_base + lr;
                    if (lr < rows_item) {
                        float u = 0.f;
#pragma unroll
                        for (int s = 0; s < TM; ++s)
                            if (s <= t) u = fmaf(sm.Tm[t][s], xs[rr][s], u);
                        st[off_u + (size_t)t * dv + row] = u;
                    }
                }
            }
            if (r0 == 0 && sp == 0) {
                for (int e = tid; e < T * DK; e += kThreads) st[e] = sm.KQ[e / DK][e % DK];
                if (tid < T) st[(size_t)T * DK + tid] = sm.G[tid];
            }
        }

        // Commit: S_L = d_{L-1} S_0 + sum_{s<L} x_s Keff_s (rollback / bad L: S_0).
        if (write_state && ok) {
            const float2 dl2 = make_float2(dl, dl);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                float2 lo[RPT], hi[RPT];
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr) {
                    lo[rr] = make_float2(S[rr][m].x, S[rr][m].y);
                    hi[rr] = make_float2(S[rr][m].z, S[rr][m].w);
                    if (L > 0) {
                        lo[rr] = __fmul2_rn(lo[rr], dl2);
                        hi[rr] = __fmul2_rn(hi[rr], dl2);
                    }
                }
#pragma unroll
                for (int s = 0; s < TM; ++s) {
                    if (s < L) {
                        const float4 ke = *reinterpret_cast<const float4*>(&sm.Keff[s][4 * (c + TPR * m)]);
                        const float2 klo = make_float2(ke.x, ke.y), khi = make_float2(ke.z, ke.w);
#pragma unroll
                        for (int rr = 0; rr < RPT; ++rr) {
                            const float2 x2 = make_float2(xs[rr][s], xs[rr][s]);
                            lo[rr] = __ffma2_rn(x2, klo, lo[rr]);
                            hi[rr] = __ffma2_rn(x2, khi, hi[rr]);
                        }
                    }
                }
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr) {
                    const int lr = r0 + grp * RPT + rr;
                    const int row = row_base + lr;
                    if (lr < rows_item)
                        __stcs(reinterpret_cast<float4*>(dst + (size_t)row * DK) + c + TPR * m,
                               make_float4(lo[rr].x, lo[rr].y, hi[rr].x, hi[rr].y));
                }
            }
        }
        // This pass's stages are free once every thread is past its reads: refill them with
        // the next item's quarters so those copies overlap the rest of this item.
        ok = !__syncthreads_or(!ok);
        if (tid == 0 && next < n_items && ok) {
            request_quarters(next, q0, q1);
            sm.refilled = q1;
        }
    }
    if (!ok) break;
    }

    // After a timed-out wait: let every copy still in flight land before the CTA's shared
    // memory is released (bounded). Stages below `refilled` hold the next item's copy.
    if (!ok && tid == 0) {
        for (int q = 0; q < nq; ++q) {
            mbar_wait_bounded(&sm.bar[q], parity, kMaxPolls);
            if (q < sm.refilled) mbar_wait_bounded(&sm.bar[q], parity ^ 1u, kMaxPolls);
        }
    }
}

template <int TM, typename InT, typename OutT>
cudaError_t launch_head_t(const VerifyArgs& a, cudaStream_t stream) {
    constexpr int RPT = TM >= 16 ? 1 : 2;
    constexpr size_t smem = sizeof(HeadSmem<TM, RPT>);
    cudaError_t e = ensure_smem_attr<gdn_verify_head_kernel<TM, RPT, InT, OutT>>((int)smem);
    if (e != cudaSuccess) return e;
    int nsm = 0;
    e = current_sm_count(&nsm);
    if (e != cudaSuccess) return e;
    // With fewer (sequence, head) items than resident CTAs, split each head's rows over 2 or
    // 4 CTAs (each redoes the small per-head algebra) so that more SMs pull state from HBM.
    VerifyArgs x = a;
    const int heads = a.B * a.Hv;
    x.row_split = 1;
    while (x.row_split < 4 && heads * x.row_split * 2 <= 2 * nsm && a.dv % (kQuarter * x.row_split * 2) == 0)
        x.row_split *= 2;
    // One CTA per item measured faster than a persistent grid that refills its stages early
    // (the hardware scheduler overlaps one CTA's algebra with the other resident CTA's
    // streaming); the kernel still loops, so a smaller grid stays correct.
    const int grid = heads * x.row_split;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gdn_verify_head_kernel<TM, RPT, InT, OutT>, x);
}

template <typename InT, typename OutT>
cudaError_t launch_head_tm(const VerifyArgs& a, cudaStream_t stream) {
    if (a.T <= 1) return launch_head_t<1, InT, OutT>(a, stream);
    if (a.T <= 2) return launch_head_t<2, InT, OutT>(a, stream);
    if (a.T <= 4) return launch_head_t<4, InT, OutT>(a, stream);
    if (a.T <= 8) return launch_head_t<8, InT, OutT>(a, stream);
    return launch_head_t<16, InT, OutT>(a, stream);
}

}  // namespace

bool head_kernel_applies(const VerifyArgs& a) {
    return a.dk == DK && a.dv >= 1 && a.dv <= kMaxRows && a.T >= 1 && a.T <= 16;
}

cudaError_t launch_verify_head(const VerifyArgs& a, cudaStream_t stream) {
    if (a.in_bf16)
        return a.out_bf16 ? launch_head_tm<__nv_bfloat16, __nv_bfloat16>(a, stream)
                          : launch_head_tm<__nv_bfloat16, float>(a, stream);
    return a.out_bf16 ? launch_head_tm<float, __nv_bfloat16>(a, stream)
                      : launch_head_tm<float, float>(a, stream);
}

}  // namespace gdn
