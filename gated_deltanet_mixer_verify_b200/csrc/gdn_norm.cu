// gdn_norm.cu -- gated RMS normalisation of the mixer's output rows, standalone:
//   y_j = x_j / sqrt(mean_j x_j^2 + eps) * w_j * silu(z_j)   (one row = one token of one head)
// ("Lithos-metal: Qwen3.8-27B on 40-core M5 Max", table "GDN mixer": gating and normalisation
// follow the recurrence inside the mixer). The tensor-core verify kernel applies the same step
// to its outputs in registers; this kernel serves every other path (decode, prefill, small
// batches) as one extra pass over the output. HBM-bound: x, z read once, y written once; one
// warp per row, 4 consecutive elements per lane, statistics in fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn_device.cuh"
#include "gdn_internal.cuh"

namespace gdn {
namespace {
using namespace dev;

constexpr int kNormWarps = 8;

template <typename T>
__device__ __forceinline__ void ld4g(const void* base, size_t i, float (&x)[4]);
template <>
__device__ __forceinline__ void ld4g<float>(const void* base, size_t i, float (&x)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
template <>
__device__ __forceinline__ void ld4g<__nv_bfloat16>(const void* base, size_t i, float (&x)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(base) + i);
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xffff0000u);
}

template <typename T>
__device__ __forceinline__ void st4g(void* base, size_t i, const float (&y)[4]);
template <>
__device__ __forceinline__ void st4g<float>(void* base, size_t i, const float (&y)[4]) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + i) = make_float4(y[0], y[1], y[2], y[3]);
}
template <>
__device__ __forceinline__ void st4g<__nv_bfloat16>(void* base, size_t i, const float (&y)[4]) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(y[0], y[1]);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(y[2], y[3]);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(base) + i) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
}

// Rows of up to 8 chunks of 128 elements are held in registers between the statistic and the
// scaling; longer rows (up to 4096) are read twice (gdn_gated_rmsnorm_long_kernel).

template <typename XT, typename ZT, typename YT, int NCH>
__global__ void __launch_bounds__(32 * kNormWarps) gdn_gated_rmsnorm_kernel(const NormArgs a) {
    const int64_t row = (int64_t)blockIdx.x * kNormWarps + (threadIdx.x >> 5);
    if (row >= a.rows) return;
    const int lane = threadIdx.x & 31;
    const size_t base = (size_t)row * a.d;
    float x[NCH][4], z[NCH][4];
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int j = 128 * c + 4 * lane;
        if (j < a.d) {
            ld4g<XT>(a.x, base + j, x[c]);
            ld4g<ZT>(a.z, base + j, z[c]);
#pragma unroll
            for (int e = 0; e < 4; ++e) ss = fmaf(x[c][e], x[c][e], ss);
        }
    }
    ss = warp_sum(ss);
    const float rs = rsqrtf(ss / (float)a.d + a.eps);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int j = 128 * c + 4 * lane;
        if (j < a.d) {
            const float4 w = __ldg(reinterpret_cast<const float4*>(a.w + j));
            const float wv[4] = {w.x, w.y, w.z, w.w};
            float y[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) y[e] = x[c][e] * rs * wv[e] * __fdividef(z[c][e], 1.f + __expf(-z[c][e]));
            st4g<YT>(a.y, base + j, y);
        }
    }
}

// Rows longer than 1024: the statistic in a first pass, then x and z again for the scaling
// (in place stays safe: each lane rereads only elements that it alone writes).
template <typename XT, typename ZT, typename YT>
__global__ void __launch_bounds__(32 * kNormWarps) gdn_gated_rmsnorm_long_kernel(const NormArgs a) {
    const int64_t row = (int64_t)blockIdx.x * kNormWarps + (threadIdx.x >> 5);
    if (row >= a.rows) return;
    const int lane = threadIdx.x & 31;
    const size_t base = (size_t)row * a.d;
    float ss = 0.f;
    for (int j = 4 * lane; j < a.d; j += 128) {
        float x[4];
        ld4g<XT>(a.x, base + j, x);
#pragma unroll
        for (int e = 0; e < 4; ++e) ss = fmaf(x[e], x[e], ss);
    }
    ss = warp_sum(ss);
    const float rs = rsqrtf(ss / (float)a.d + a.eps);
    for (int j = 4 * lane; j < a.d; j += 128) {
        float x[4], z[4], y[4];
        ld4g<XT>(a.x, base + j, x);
        ld4g<ZT>(a.z, base + j, z);
        const float4 w = __ldg(reinterpret_cast<const float4*>(a.w + j));
        const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) y[e] = x[e] * rs * wv[e] * __fdividef(z[e], 1.f + __expf(-z[e]));
        st4g<YT>(a.y, base + j, y);
    }
}

template <typename XT, typename ZT, typename YT>
cudaError_t launch_xzy(const NormArgs& a, cudaStream_t stream) {
    const dim3 grid((unsigned)((a.rows + kNormWarps - 1) / kNormWarps));
    const int nch = (a.d + 127) / 128;
    if (nch <= 1) gdn_gated_rmsnorm_kernel<XT, ZT, YT, 1><<<grid, 32 * kNormWarps, 0, stream>>>(a);
    else if (nch <= 2) gdn_gated_rmsnorm_kernel<XT, ZT, YT, 2><<<grid, 32 * kNormWarps, 0, stream>>>(a);
    else if (nch <= 8) gdn_gated_rmsnorm_kernel<XT, ZT, YT, 8><<<grid, 32 * kNormWarps, 0, stream>>>(a);
    else gdn_gated_rmsnorm_long_kernel<XT, ZT, YT><<<grid, 32 * kNormWarps, 0, stream>>>(a);
    return cudaGetLastError();
}

template <typename XT, typename ZT>
cudaError_t launch_xz(const NormArgs& a, cudaStream_t stream) {
    return a.y_bf16 ? launch_xzy<XT, ZT, __nv_bfloat16>(a, stream) : launch_xzy<XT, ZT, float>(a, stream);
}

template <typename XT>
cudaError_t launch_x(const NormArgs& a, cudaStream_t stream) {
    return a.z_bf16 ? launch_xz<XT, __nv_bfloat16>(a, stream) : launch_xz<XT, float>(a, stream);
}

}  // namespace

cudaError_t launch_gated_rmsnorm(const NormArgs& a, cudaStream_t stream) {
    if (a.rows == 0) return cudaSuccess;
    return a.x_bf16 ? launch_x<__nv_bfloat16>(a, stream) : launch_x<float>(a, stream);
}

}  // namespace gdn
