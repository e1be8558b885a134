// gdn_conv.cu -- causal short convolution over the mixer's q, k, v with the filter layer's
// short history, rewound to the accepted prefix at device-resident accept counts.
//
// The short history a small filter layer keeps is one of the three structures brought back
// in line with the accepted tokens after every verify block, with the key-value cache and the
// recurrent state ("Qwen 3.8 27B mac m5: 200 tok/s, audited", section "How does DSpark
// speculative decoding create more than one token per read?"). The page gives no width or
// activation; the plain reading built here: one filter of K taps per channel,
//   y_t = silu(sum_{i<K} w[c][i] xc[t + i]),  xc = [history (K-1 inputs, oldest first), x],
// and after acceptance of L tokens the history becomes xc[L .. L + K - 2].
//
// Channels run [q (H_k d_k) | k (H_k d_k) | v (H_v d_v)]; one token's row of each tensor is
// contiguous. A CTA owns 256 channels of one sequence over a tile of tokens and stages its rows
// in shared memory with bulk asynchronous copies, so that every load of the grid is in flight
// at once (registers hold no staged data); every input element is read once (plus a K-1 row
// halo per tile) and every output written once: HBM-bound.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.cuh"

namespace gdn {
namespace {
using namespace dev;

constexpr int kConvThreads = 128;

// The tensor holding channel c (a multiple of 8) and the column of c inside its token row.
struct Chan {
    const void* in;
    void* out;
    int col;
    int width;
};

__device__ __forceinline__ Chan channel(const ConvArgs& a, int c) {
    if (c < a.Cq) return {a.q, a.q_out, c, a.Cq};
    if (c < 2 * a.Cq) return {a.k, a.k_out, c - a.Cq, a.Cq};
    return {a.v, a.v_out, c - 2 * a.Cq, a.C - 2 * a.Cq};
}

// Four consecutive elements (i a multiple of 4; 8 bytes for bf16, 16 for fp32). NC: through
// the read-only path (inputs the launch never writes); otherwise a plain coherent load (the
// history may be rewritten in place by the thread that reads it).
template <typename T, bool NC>
__device__ __forceinline__ void ld4(const void* base, size_t i, float (&x)[4]);
template <>
__device__ __forceinline__ void ld4<float, true>(const void* base, size_t i, float (&x)[4]) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
template <>
__device__ __forceinline__ void ld4<float, false>(const void* base, size_t i, float (&x)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
__device__ __forceinline__ void unpack_bf16x4(uint2 u, float (&x)[4]) {
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xffff0000u);
}
template <>
__device__ __forceinline__ void ld4<__nv_bfloat16, true>(const void* base, size_t i, float (&x)[4]) {
    unpack_bf16x4(__ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(base) + i)), x);
}
template <>
__device__ __forceinline__ void ld4<__nv_bfloat16, false>(const void* base, size_t i, float (&x)[4]) {
    unpack_bf16x4(*reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(base) + i), x);
}

template <typename T>
__device__ __forceinline__ void st4(void* base, size_t i, const float (&y)[4]);
template <>
__device__ __forceinline__ void st4<float>(void* base, size_t i, const float (&y)[4]) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + i) = make_float4(y[0], y[1], y[2], y[3]);
}
template <>
__device__ __forceinline__ void st4<__nv_bfloat16>(void* base, size_t i, const float (&y)[4]) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(y[0], y[1]);   // .x = the lower address
    const __nv_bfloat162 hi = __floats2bfloat162_rn(y[2], y[3]);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(base) + i) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
}

// xc row r of sequence b, channels c .. c + 3: history row r (r < K-1) or token r - (K-1).
template <int K, typename InT>
__device__ __forceinline__ void load_xc(const ConvArgs& a, const Chan& ch, int b, int c, int r, float (&x)[4]) {
    if (r < K - 1)
        ld4<InT, false>(a.hist_in, ((size_t)b * (K - 1) + r) * a.C + c, x);
    else
        ld4<InT, true>(ch.in, ((size_t)b * a.T + (r - (K - 1))) * ch.width + ch.col, x);
}

// The accepted count of sequence b (all T without counts); an out-of-range count keeps the
// old history (L = 0) and sets status bit 1 once per sequence.
__device__ __forceinline__ int accepted(const ConvArgs& a, int b, int c) {
    int L = a.accept_len ? a.accept_len[b] : a.T;
    if (L < 0 || L > a.T) {
        if (c == 0 && a.status_word) atomicOr(a.status_word, kStatusBadAccept);
        L = 0;
    }
    return L;
}

template <int K, typename InT>
__device__ __forceinline__ void store_hist(const ConvArgs& a, int b, int c, const float (&hn)[K - 1][4]) {
#pragma unroll
    for (int j = 0; j < K - 1; ++j) st4<InT>(a.hist_out, ((size_t)b * (K - 1) + j) * a.C + c, hn[j]);
}

constexpr int kConvChannels = 256;   // channels per CTA (4 per thread, 64 threads)
constexpr int kConvTile = 32;        // tokens per CTA; T <= 32 is one tile
constexpr uint32_t kConvMaxPolls = 1u << 24;

// Shared memory of one CTA: the xc rows of its tile ([K - 1 + tile][256] in InT), then the taps
// ([256][K] fp32), then the mbarrier. Sized on the host with the same formula.
__host__ __device__ constexpr size_t conv_rows_bytes(int K, int tile, size_t el) {
    return (size_t)(K - 1 + tile) * kConvChannels * el;
}
__host__ __device__ constexpr size_t conv_smem_bytes(int K, int tile, size_t el) {
    return conv_rows_bytes(K, tile, el) + (size_t)kConvChannels * K * 4 + 16;
}

// grid (ceil(C / 256), token tiles, B), 64 threads. The CTA stages the rows it needs -- the
// K - 1 rows before its tile (the history for the first tile) and the tile's inputs -- and
// its 256 x K taps in shared memory with bulk asynchronous copies on one mbarrier: a token
// row's 256 channels are up to three contiguous pieces (the q | k | v boundaries), a history
// row is one. Then thread i convolves channels 4i .. 4i + 3 from shared memory. With one tile
// the same launch rewinds the history from the staged rows: the copies have read every old
// history row before any thread writes, and each history element belongs to one CTA, so in
// place is safe. Several tiles leave the rewind to gdn_conv_rewind_kernel.
template <int K, typename InT>
__global__ void __launch_bounds__(64) gdn_short_conv_kernel(const ConvArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int tid = threadIdx.x;
    const int c0 = blockIdx.x * kConvChannels;
    const int nc = min(kConvChannels, a.C - c0);
    const int b = blockIdx.z;
    const int t0 = blockIdx.y * a.tile;
    const int t1 = min(t0 + a.tile, a.T);
    const int rows = K - 1 + (t1 - t0);
    constexpr size_t el = sizeof(InT);
    InT* xs = reinterpret_cast<InT*>(smem);
    float* ws = reinterpret_cast<float*>(smem + conv_rows_bytes(K, a.tile, el));
    uint64_t* bar = reinterpret_cast<uint64_t*>(ws + kConvChannels * K);

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
        mbar_arrive_expect_tx(bar, (uint32_t)(((size_t)rows * nc * el) + (size_t)nc * K * 4));
    }
    __syncthreads();
    for (int r = tid; r < rows; r += 64) {
        const int xr = t0 + r;   // xc row: history row xr, or token xr - (K - 1)
        InT* dst = xs + (size_t)r * kConvChannels;
        if (xr < K - 1) {
            bulk_g2s(dst, static_cast<const InT*>(a.hist_in) + ((size_t)b * (K - 1) + xr) * a.C + c0,
                     (uint32_t)(nc * el), bar);
        } else {
            const int tok = xr - (K - 1);
            const int lo[3] = {0, a.Cq, 2 * a.Cq};
            const int hi[3] = {a.Cq, 2 * a.Cq, a.C};
            const void* src[3] = {a.q, a.k, a.v};
#pragma unroll
            for (int p = 0; p < 3; ++p) {
                const int s = max(c0, lo[p]), e = min(c0 + nc, hi[p]);
                if (s < e)
                    bulk_g2s(dst + (s - c0),
                             static_cast<const InT*>(src[p]) + ((size_t)b * a.T + tok) * (hi[p] - lo[p]) + (s - lo[p]),
                             (uint32_t)((e - s) * el), bar);
            }
        }
    }
    if (tid == 63) bulk_g2s(ws, a.w + (size_t)c0 * K, (uint32_t)(nc * K * 4), bar);
    const bool landed = mbar_wait_bounded(bar, 0, kConvMaxPolls);
    if (!__syncthreads_and(landed)) {
        if (tid == 0) {
            if (a.status_word) atomicOr(a.status_word, kStatusWaitTimeout);
            mbar_wait_bounded(bar, 0, kConvMaxPolls);   // let the copies land before exiting
        }
        return;
    }

    const int cl = 4 * tid;   // channels c0 + cl .. + 3
    if (cl >= nc) return;
    float w[K][4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int i = 0; i < K; ++i) w[i][e] = ws[(cl + e) * K + i];
    const Chan ch = channel(a, c0 + cl);
    float xw[K - 1][4];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) ld4<InT, false>(xs, (size_t)j * kConvChannels + cl, xw[j]);
    for (int r = K - 1; r < rows; ++r) {
        float x[4];
        ld4<InT, false>(xs, (size_t)r * kConvChannels + cl, x);
        float y[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float z = w[K - 1][e] * x[e];
#pragma unroll
            for (int j = 0; j < K - 1; ++j) z = fmaf(w[j][e], xw[j][e], z);
            y[e] = __fdividef(z, 1.f + __expf(-z));
        }
        st4<InT>(ch.out, ((size_t)b * a.T + t0 + r - (K - 1)) * ch.width + ch.col, y);
#pragma unroll
        for (int j = 0; j < K - 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) xw[j][e] = xw[j + 1][e];
#pragma unroll
        for (int e = 0; e < 4; ++e) xw[K - 2][e] = x[e];
    }
    if (a.fused_hist) {   // one tile (t0 = 0): staged row r is xc row r
        const int L = accepted(a, b, c0 + cl);
#pragma unroll
        for (int j = 0; j < K - 1; ++j) {
            float h[4];
            ld4<InT, false>(xs, (size_t)(L + j) * kConvChannels + cl, h);
            st4<InT>(a.hist_out, ((size_t)b * (K - 1) + j) * a.C + c0 + cl, h);
        }
    }
}

// grid (channel quads / 128, 1, B): the history rewind alone (two-phase commit of the history,
// or after a convolution of more than 8 tokens). Rows are read before any is written.
template <int K, typename InT>
__global__ void __launch_bounds__(kConvThreads) gdn_conv_rewind_kernel(const ConvArgs a) {
    const int c = 4 * (blockIdx.x * kConvThreads + threadIdx.x);
    if (c >= a.C) return;
    const int b = blockIdx.z;
    const Chan ch = channel(a, c);
    const int L = accepted(a, b, c);
    float hn[K - 1][4];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) load_xc<K, InT>(a, ch, b, c, L + j, hn[j]);
    store_hist<K, InT>(a, b, c, hn);
}

template <int K, typename InT>
cudaError_t launch_k(ConvArgs a, cudaStream_t stream) {
    const bool outputs = a.q_out != nullptr;
    const int tile = a.T <= kConvTile ? a.T : kConvTile;
    const int ntiles = (a.T + tile - 1) / tile;
    a.tile = tile;
    a.fused_hist = a.hist_out != nullptr && ntiles == 1;
    if (outputs) {
        const size_t smem = conv_smem_bytes(K, tile, sizeof(InT));   // <= 40 KB: no opt-in needed
        gdn_short_conv_kernel<K, InT><<<dim3((a.C + kConvChannels - 1) / kConvChannels, ntiles, a.B), 64, smem,
                                        stream>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.hist_out && !(outputs && a.fused_hist)) {
        const int quads = a.C / 4;
        gdn_conv_rewind_kernel<K, InT><<<dim3((quads + kConvThreads - 1) / kConvThreads, 1, a.B), kConvThreads, 0,
                                         stream>>>(a);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

template <typename InT>
cudaError_t launch_t(const ConvArgs& a, int K, cudaStream_t stream) {
    switch (K) {
        case 2: return launch_k<2, InT>(a, stream);
        case 3: return launch_k<3, InT>(a, stream);
        case 4: return launch_k<4, InT>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_short_conv(const ConvArgs& a, int K, bool bf16, cudaStream_t stream) {
    return bf16 ? launch_t<__nv_bfloat16>(a, K, stream) : launch_t<float>(a, K, stream);
}

}  // namespace gdn
