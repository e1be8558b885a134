// gdn_accept.cu -- device-side acceptance of a verify block: greedy matching or exact
// speculative sampling, producing the accept counts the mixer commits at and the next token,
// so that verify -> accept -> commit stays on the GPU.
//
// Rule ("Qwen 3.8 27B mac m5: 200 tok/s, audited", section "How does DSpark speculative
// decoding create more than one token per read?"): row 0 of a block is the anchor, rows
// 1..T-1 the drafts. Greedy keeps draft t+1 only if it is the target's argmax at row t
// (lowest index among equal maxima); sampled mode keeps it when u * q_t(d) < p_t(d), i.e. with
// probability min(1, p / q), p_t = softmax(target_t / tau), q_t = softmax(draft_t / tau). After
// n leading survivors: accept_len = n + 1; the next token is argmax p_n (greedy), else a draw
// with u_0 from the residual max(0, p_n - q_n) (n < T-1) or from p_{T-1} (all survived).
//
// Kernel 1 (one CTA per logit row, a sequence's target rows then its draft rows, sequences in
// order, so that sequences are finished one after another): streams the row once with
// 16-byte loads, keeping the maximum and its first index (greedy) or the online maximum and
// sum of 2^(x log2(e) / tau - max) (sampled). The last CTA to finish a sequence's rows (a
// fence, then an atomic counter: nobody waits) finds n, writes accept_len (and the greedy
// next token) and raises the sequence's flag. Kernel 2 (sampled; 8 CTAs per sequence): tile
// sums (256 logits a tile) of the residual over row n; the last CTA of the sequence draws the
// token by inverse CDF, first over the tile sums, then inside one tile with a warp scan.
// Kernel 2 is a programmatic dependent of kernel 1: it is launched once every CTA of kernel 1
// has started (each releases it at entry), and each of its CTAs waits for its sequence's flag
// rather than for the whole of kernel 1, so that the draws of the sequences already finished
// overlap the rows still streaming. Kernel 1 never waits and all of its CTAs have started,
// so every flag is raised and every wait ends (it is bounded all the same, with a status
// bit). Run after kernel 1 in plain stream order, the draw took 28% of the call's time for
// 10% of its bytes. (Measured and slower: one persistent kernel doing both phases, over equal
// contiguous shares of the logits, over shares fed by bulk copies through a shared-memory
// ring, or over a list of quarter-row and draw items walked in grid strides or taken by an
// atomic ticket; each paid a row piece's fixed latency once per item in series.)
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.cuh"

namespace gdn {
namespace {
using namespace dev;

constexpr int kRowThreads = 512;
constexpr int kTile = 256;         // logits per tile of the residual draw (8 per lane of a warp)
constexpr int kSplit = 8;          // CTAs per sequence in the residual pass
constexpr int kSplitThreads = 256;
constexpr int kGreedyPadBytes = 80 * 1024;   // two row CTAs per SM in greedy calls (see launch_accept)
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kMaxPolls = 1u << 20;   // bound of a draw CTA's wait for its sequence (~0.1-1 s)

using RowStat = AcceptRowStat;

// Eight consecutive logits kept raw while their loads are in flight (bf16 pairs, not fp32),
// widened where they are used.
template <typename T>
struct Raw8;
template <>
struct Raw8<float> {
    float4 a, b;
};
template <>
struct Raw8<__nv_bfloat16> {
    uint4 u;
};
__device__ __forceinline__ void ld8raw(const float* p, Raw8<float>& r) {
    r.a = __ldcs(reinterpret_cast<const float4*>(p));
    r.b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
}
__device__ __forceinline__ void ld8raw(const __nv_bfloat16* p, Raw8<__nv_bfloat16>& r) {
    r.u = __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void widen8(const Raw8<float>& r, float (&x)[8]) {
    x[0] = r.a.x; x[1] = r.a.y; x[2] = r.a.z; x[3] = r.a.w;
    x[4] = r.b.x; x[5] = r.b.y; x[6] = r.b.z; x[7] = r.b.w;
}
__device__ __forceinline__ void widen8(const Raw8<__nv_bfloat16>& r, float (&x)[8]) {
    const uint32_t w[4] = {r.u.x, r.u.y, r.u.z, r.u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[2 * e] = __uint_as_float(w[e] << 16);
        x[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}
__device__ __forceinline__ void fill8(Raw8<float>& r) {
    r.a = r.b = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
}
__device__ __forceinline__ void fill8(Raw8<__nv_bfloat16>& r) {
    const uint32_t ninf = 0xff80ff80u;   // two bf16 -inf
    r.u = make_uint4(ninf, ninf, ninf, ninf);
}

template <typename T>
__device__ __forceinline__ float ld1l(const T* p, int64_t i) {
    return to_f(p[i]);
}

// (value, index) maximum with ties to the lower index.
__device__ __forceinline__ void better(float& v, int& i, float v2, int i2) {
    if (v2 > v || (v2 == v && i2 < i)) {
        v = v2;
        i = i2;
    }
}

// Online (max, sum) of base-2 exponentials: merge (m2, s2) into (m, s).
__device__ __forceinline__ void merge_ms(float& m, float& s, float m2, float s2) {
    const float mn = fmaxf(m, m2);
    if (mn == -INFINITY) return;
    s = s * exp2_approx(m - mn) + s2 * exp2_approx(m2 - mn);
    m = mn;
}

// The decisions of sequence b, one draft per lane (warp-wide call): greedy compares the draft
// with the row's first argmax; sampled tests u * q < p with p, q from the row statistics. n is
// the length of the leading run of survivors; lane 0 writes accept_len = n + 1 (and the greedy
// next token) and keeps n for the draw.
template <typename LT>
__device__ void decide(const AcceptArgs& a, int b, int lane) {
    bool ok = false;
    const int t = lane;
    if (t + 1 < a.T) {
        const int d = a.tokens[(int64_t)b * a.T + t + 1];
        const RowStat* st = a.stats;
        if (!a.sampled) {
            ok = d == __ldcg(&st[(int64_t)b * a.T + t].arg);
        } else if (d >= 0 && d < a.V) {
            const float c = kLog2e / a.tau;
            const int64_t pr = (int64_t)b * a.T + t;
            const int64_t qr = (int64_t)a.B * a.T + (int64_t)b * (a.T - 1) + t;
            const float lp = ld1l(static_cast<const LT*>(a.target), pr * a.V + d);
            const float lq = ld1l(static_cast<const LT*>(a.draft), ((int64_t)b * (a.T - 1) + t) * a.V + d);
            const float p = exp2_approx(lp * c - __ldcg(&st[pr].m)) / __ldcg(&st[pr].s);
            const float q = exp2_approx(lq * c - __ldcg(&st[qr].m)) / __ldcg(&st[qr].s);
            ok = a.u[(int64_t)b * a.T + t + 1] * q < p;
        }
    }
    const unsigned bits = __ballot_sync(kFull, ok);
    const unsigned full = (a.T - 1 >= 32) ? kFull : ((1u << (a.T - 1)) - 1u);
    const int n = ((bits & full) == full) ? a.T - 1 : __ffs(~bits) - 1;
    if (lane == 0) {
        a.accept_len[b] = n + 1;
        a.nsurv[b] = n;
        if (!a.sampled) a.next_token[b] = __ldcg(&a.stats[(int64_t)b * a.T + n].arg);
    }
}

__device__ __forceinline__ uint32_t ld_acquire(const int* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// One CTA per logit row (a sequence's target rows, then its draft rows): the row streamed
// once, four 8-logit groups per thread in flight, the next four issued before the current
// four are used (addresses clamped into the row, values past its end masked, so that no
// branch sits between the loads). The last row of a sequence
// (fence, then an atomic counter: nothing waits) has warp 0 decide and raise the flag.
template <typename LT>
__global__ void __launch_bounds__(kRowThreads) gdn_accept_rows_kernel(const AcceptArgs a) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the draw kernel may launch
    const int rows_per_seq = a.sampled ? 2 * a.T - 1 : a.T;
    const int b = (int)(blockIdx.x / rows_per_seq), k = (int)(blockIdx.x % rows_per_seq);
    const int64_t ntarget = (int64_t)a.B * a.T;
    const int64_t r = k < a.T ? (int64_t)b * a.T + k : ntarget + (int64_t)b * (a.T - 1) + (k - a.T);
    const LT* row = r < ntarget ? static_cast<const LT*>(a.target) + r * a.V
                                : static_cast<const LT*>(a.draft) + (r - ntarget) * a.V;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float c = kLog2e / a.tau;
    float m = -INFINITY, s = 0.f;
    int arg = 0x7fffffff;
    Raw8<LT> nx[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) ld8raw(row + min(8 * tid + g * 8 * kRowThreads, a.V - 8), nx[g]);
    for (int base = 8 * tid; base < a.V; base += 4 * 8 * kRowThreads) {
        Raw8<LT> xr[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) xr[g] = nx[g];
#pragma unroll
        for (int g = 0; g < 4; ++g) ld8raw(row + min(base + 4 * 8 * kRowThreads + g * 8 * kRowThreads, a.V - 8), nx[g]);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int i = base + g * 8 * kRowThreads;
            if (i >= a.V) continue;
            float x[8];
            widen8(xr[g], x);
            if (!a.sampled) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (x[e] > m) {   // indices rise within a thread: strict > keeps the first
                        m = x[e];
                        arg = i + e;
                    }
            } else {
                // one exponential per logit: the running sum is rescaled only when the running
                // maximum grows (rarely, after a thread's first groups)
                float lm = m;
#pragma unroll
                for (int e = 0; e < 8; ++e) lm = fmaxf(lm, x[e] * c);
                if (lm > m) {
                    s *= exp2_approx(m - lm);   // 0 when m is still -inf
                    m = lm;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) s += exp2_approx(x[e] * c - m);
            }
        }
    }
    __shared__ float red_m[kRowThreads / 32], red_s[kRowThreads / 32];
    __shared__ int red_i[kRowThreads / 32];
    __shared__ bool last;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float m2 = __shfl_xor_sync(kFull, m, off);
        const float s2 = __shfl_xor_sync(kFull, s, off);
        const int i2 = __shfl_xor_sync(kFull, arg, off);
        if (!a.sampled) better(m, arg, m2, i2);
        else merge_ms(m, s, m2, s2);
    }
    if (lane == 0) {
        red_m[warp] = m;
        red_s[warp] = s;
        red_i[warp] = arg;
    }
    __syncthreads();
    if (tid == 0) {
        for (int w = 1; w < kRowThreads / 32; ++w) {
            if (!a.sampled) better(m, arg, red_m[w], red_i[w]);
            else merge_ms(m, s, red_m[w], red_s[w]);
        }
        RowStat* st = a.stats + r;
        st->m = m;
        st->s = s;
        st->arg = arg;
        __threadfence();   // the statistics are visible before this row is counted
        last = atomicAdd(&a.counters[b], 1) == rows_per_seq - 1;
    }
    __syncthreads();
    if (!last || warp != 0) return;
    __threadfence();
    decide<LT>(a, b, lane);
    if (lane == 0) {
        __threadfence();
        st_release(&a.decided[b], 1);
    }
}

// Logits j .. j+7 of the target row (and the draft row) as raw values; -inf past the row.
template <typename LT>
__device__ __forceinline__ void load_pair(const LT* pr, const LT* qr, int j, int V, Raw8<LT>& x, Raw8<LT>& y) {
    fill8(x);
    fill8(y);
    if (j < V) {
        ld8raw(pr + j, x);
        if (qr) ld8raw(qr + j, y);
    }
}

// Residual (or target) weights from raw logits and the row statistics (pi, qi: the reciprocals
// of the row sums).
template <typename LT>
__device__ __forceinline__ void weights_of(const Raw8<LT>& xr, const Raw8<LT>& yr, bool resid, float c, float pm,
                                           float pi, float qm, float qi, float (&w)[8]) {
    float x[8], y[8];
    widen8(xr, x);
    widen8(yr, y);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        float v = exp2_approx(x[e] * c - pm) * pi;
        if (resid) v = fmaxf(v - exp2_approx(y[e] * c - qm) * qi, 0.f);
        w[e] = x[e] == -INFINITY ? 0.f : v;
    }
}

constexpr int kMaxTiles = 1024;   // V <= 2^18

// grid (B, kSplit): tile sums of row n's residual, 4 tiles in flight per warp; the last CTA of
// the sequence stages all tile sums in shared memory and draws the token by inverse CDF.
template <typename LT>
__global__ void __launch_bounds__(kSplitThreads) gdn_accept_draw_kernel(const AcceptArgs a) {
    const int b = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ int ok_s;
    if (tid == 0) {   // the sequence's counts (see the note at the top)
        uint32_t polls = 0;
        int ok = 1;
        while (ld_acquire(&a.decided[b]) == 0) {
            if (++polls > (a.max_polls ? a.max_polls : kMaxPolls)) {
                ok = 0;
                break;
            }
            __nanosleep(128);
        }
        ok_s = ok;
    }
    __syncthreads();
    if (!ok_s) {
        if (tid == 0) {
            if (a.status_word) atomicOr(a.status_word, kStatusWaitTimeout);
            a.next_token[b] = 0;
        }
        return;
    }
    const int n = __ldcg(&a.nsurv[b]);
    const int64_t prow = (int64_t)b * a.T + n;
    const LT* pr = static_cast<const LT*>(a.target) + prow * a.V;
    const LT* qr = nullptr;
    float qm = 0.f, qs = 1.f;
    if (n < a.T - 1) {
        const int64_t q = (int64_t)a.B * a.T + (int64_t)b * (a.T - 1) + n;
        qr = static_cast<const LT*>(a.draft) + ((int64_t)b * (a.T - 1) + n) * a.V;
        qm = __ldcg(&a.stats[q].m);
        qs = __ldcg(&a.stats[q].s);
    }
    const bool resid = qr != nullptr;
    const float pm = __ldcg(&a.stats[prow].m), pi = 1.f / __ldcg(&a.stats[prow].s);
    qs = 1.f / qs;   // from here on the reciprocal
    const float c = kLog2e / a.tau;
    const int ntiles = (a.V + kTile - 1) / kTile;
    float* tsum = a.tiles + (int64_t)b * ntiles;
    constexpr int kStride = kSplit * (kSplitThreads / 32);   // tiles between a warp's iterations
    for (int t0 = blockIdx.y + kSplit * warp; t0 < ntiles; t0 += 4 * kStride) {
        Raw8<LT> x[4], y[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) load_pair<LT>(pr, qr, (t0 + k * kStride) * kTile + 8 * lane, a.V, x[k], y[k]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int tile = t0 + k * kStride;
            float w[8];
            weights_of(x[k], y[k], resid, c, pm, pi, qm, qs, w);
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc += w[e];
            acc = warp_sum(acc);
            if (lane == 0 && tile < ntiles) tsum[tile] = acc;
        }
    }
    __shared__ bool last;
    __shared__ float sts[kMaxTiles];
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        last = atomicAdd(&a.counters[a.B + b], 1) == kSplit - 1;
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int t = tid; t < ntiles; t += kSplitThreads) sts[t] = __ldcg(&tsum[t]);
    __syncthreads();
    if (warp != 0) return;
    // Warp 0: the total and the tile holding u_0 * total (lane L sums a contiguous range of
    // tiles), then the logit inside that tile.
    const int per = (ntiles + 31) / 32;
    const int r0 = min(lane * per, ntiles), r1 = min(r0 + per, ntiles);
    float mine = 0.f;
    for (int t = r0; t < r1; ++t) mine += sts[t];
    float incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float v = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += v;
    }
    const float total = __shfl_sync(kFull, incl, 31);
    const float target = a.u[(int64_t)b * a.T] * total;
    const unsigned hit = __ballot_sync(kFull, incl > target && mine > 0.f);
    const bool fallback = hit == 0;   // rounding put u_0 * total at the very end
    int tile = -1;
    float before = 0.f;
    if (!fallback) {
        const int L = __ffs(hit) - 1;
        if (lane == L) {
            float cum = incl - mine;
            for (int t = r0; t < r1; ++t) {
                if (cum + sts[t] > target && sts[t] > 0.f) {
                    tile = t;
                    break;
                }
                cum += sts[t];
            }
            if (tile < 0)
                for (int t = r1 - 1; t >= r0; --t)
                    if (sts[t] > 0.f) {
                        tile = t;
                        break;
                    }
            before = cum;
        }
        tile = __shfl_sync(kFull, tile, L);
        before = __shfl_sync(kFull, before, L);
    } else {
        int lt = -1;
        for (int t = ntiles - 1 - lane; t >= 0; t -= 32)
            if (sts[t] > 0.f) {
                lt = t;
                break;
            }
        tile = __reduce_max_sync(kFull, lt);
    }
    if (tile < 0) {
        if (lane == 0) a.next_token[b] = 0;
        return;
    }
    const int j = tile * kTile + 8 * lane;
    Raw8<LT> x, y;
    float w[8];
    load_pair<LT>(pr, qr, j, a.V, x, y);
    weights_of(x, y, resid, c, pm, pi, qm, qs, w);
    float mine2 = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) mine2 += w[e];
    float incl2 = mine2;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float v = __shfl_up_sync(kFull, incl2, off);
        if (lane >= off) incl2 += v;
    }
    // The first logit whose running mass passes the target; else the tile's last positive one.
    int found = 0x7fffffff, lastpos = -1;
    float cum = before + incl2 - mine2;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        cum += w[e];
        if (w[e] > 0.f) {
            if (cum > target && found == 0x7fffffff) found = j + e;
            lastpos = j + e;
        }
    }
    const int first = __reduce_min_sync(kFull, found);
    const int lastp = __reduce_max_sync(kFull, lastpos);
    if (lane == 0) a.next_token[b] = (!fallback && first != 0x7fffffff) ? first : (lastp >= 0 ? lastp : 0);
}

// A flag that nothing raises, for the wait self-test.
__device__ int g_never_raised = 0;

}  // namespace

cudaError_t launch_accept_wait_selftest(int32_t* status_word, int32_t* next_token, uint32_t polls,
                                        cudaStream_t stream) {
    // One sequence whose flag never rises: every draw CTA gives up after `polls` polls, sets
    // the wait-timeout bit and writes next token 0, touching nothing else.
    AcceptArgs a = {};
    a.B = 1;
    a.T = 2;
    a.V = 8;
    a.bf16 = true;
    a.sampled = true;
    a.tau = 1.f;
    a.status_word = status_word;
    a.next_token = next_token;
    a.max_polls = polls;
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&a.decided), g_never_raised);
    if (e != cudaSuccess) return e;
    gdn_accept_draw_kernel<__nv_bfloat16><<<dim3(1, kSplit), kSplitThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

size_t accept_workspace_bytes(int B, int T, int V, bool sampled) {
    const size_t rows = (size_t)B * T + (sampled ? (size_t)B * (T - 1) : 0);
    const size_t ntiles = ((size_t)V + kTile - 1) / kTile;
    return rows * sizeof(RowStat) /* stats */ + (size_t)3 * B * 4 /* counters, flags */ + (size_t)B * 4 /* n */ +
           (sampled ? (size_t)B * ntiles * 4 : 0) + 64;
}

cudaError_t launch_accept(AcceptArgs a, void* workspace, cudaStream_t stream) {
    // Workspace: row statistics, the counters (rows done per sequence, draw CTAs done per
    // sequence) and the sequences' flags, n per sequence, the tile sums.
    const size_t rows = (size_t)a.B * a.T + (a.sampled ? (size_t)a.B * (a.T - 1) : 0);
    unsigned char* w = static_cast<unsigned char*>(workspace);
    a.stats = reinterpret_cast<RowStat*>(w);
    w += rows * sizeof(RowStat);
    a.counters = reinterpret_cast<int*>(w);
    a.decided = a.counters + 2 * (size_t)a.B;
    w += (size_t)3 * a.B * 4;
    a.nsurv = reinterpret_cast<int*>(w);
    w += (size_t)a.B * 4;
    a.tiles = reinterpret_cast<float*>(w);
    cudaError_t e = cudaMemsetAsync(a.counters, 0, (size_t)3 * a.B * 4, stream);
    if (e != cudaSuccess) return e;
    // Greedy calls reserve shared memory they do not use, so that at most two row CTAs share an
    // SM whatever the register allocation: at three, the 512 rows of a 64 x 8 block make 1.15
    // waves on 148 SMs and the second runs nearly empty (0.047 against 0.041 ms, measured when
    // the kernel took 40 registers; it now takes 58, which also allows two).
    const int pad = a.sampled ? 0 : kGreedyPadBytes;
    if (!a.sampled) {
        e = a.bf16 ? ensure_smem_attr<gdn_accept_rows_kernel<__nv_bfloat16>>(kGreedyPadBytes)
                   : ensure_smem_attr<gdn_accept_rows_kernel<float>>(kGreedyPadBytes);
        if (e != cudaSuccess) return e;
    }
    if (a.bf16) gdn_accept_rows_kernel<__nv_bfloat16><<<(unsigned)rows, kRowThreads, pad, stream>>>(a);
    else gdn_accept_rows_kernel<float><<<(unsigned)rows, kRowThreads, pad, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess || !a.sampled) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.B, kSplit);
    cfg.blockDim = dim3(kSplitThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return a.bf16 ? cudaLaunchKernelEx(&cfg, gdn_accept_draw_kernel<__nv_bfloat16>, a)
                  : cudaLaunchKernelEx(&cfg, gdn_accept_draw_kernel<float>, a);
}

}  // namespace gdn
