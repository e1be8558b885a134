// gdn_device.cuh -- device helpers shared by the mixer kernels: typed loads / stores,
// warp reductions, the gate non-linearities, and thin wrappers over the sm_90+/sm_100
// asynchronous bulk-copy and mbarrier instructions (inline PTX).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {
namespace dev {

constexpr unsigned kFull = 0xffffffffu;

// Status bits OR-ed into the caller's status word (see include/gdn.h).
constexpr int kStatusBadAccept = 1;
constexpr int kStatusWaitTimeout = 2;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ float ld_in(const void* base, size_t i) {
    return to_f(reinterpret_cast<const T*>(base)[i]);
}

// Eight consecutive input elements starting at element i (i a multiple of 8, base 16-byte
// aligned): one 16-byte load for bf16, two for fp32.
template <typename T>
__device__ __forceinline__ void ld8(const void* base, size_t i, float (&x)[8]);
template <>
__device__ __forceinline__ void ld8<float>(const void* base, size_t i, float (&x)[8]) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
template <>
__device__ __forceinline__ void ld8<__nv_bfloat16>(const void* base, size_t i, float (&x)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(base) + i));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[2 * e] = __uint_as_float(w[e] << 16);
        x[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
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

// Sum over aligned groups of W consecutive lanes (W a power of two <= 32).
template <int W>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int off = W / 2; off >= 1; off >>= 1) x += __shfl_xor_sync(kFull, x, off);
    return x;
}

// 2^x by the hardware approximation (ex2.approx.ftz: relative error about 2^-22, subnormal
// results flushed to zero).
__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Named barrier `id` (1..15) over the first `nthreads` threads of the block (a multiple of 32).
__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }

// Halving butterfly over the lanes of an aligned group (lane bits below 2*OFF). On return a
// lane whose in-group index is c holds, in v[0..max(CNT/W,1)), the fully reduced values whose
// original indices start at c*CNT/W (CNT >= W) or equal c/(W/CNT) (CNT < W), W = 2*OFF.
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

// ---------------------------------------------------------------- async bulk copy + mbarrier

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make initialised barriers visible to the asynchronous (bulk-copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Global -> shared bulk copy (both addresses 16-byte aligned, bytes a multiple of 16); the
// completed bytes are counted on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// One arrival on `bar` (release semantics at CTA scope).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Shared -> global bulk copy (both addresses 16-byte aligned, bytes a multiple of 16), tracked
// by this thread's bulk async-groups; bulk_commit() closes the group.
__device__ __forceinline__ void bulk_s2g(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk group of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until every committed bulk group of this thread has completed (writes performed).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Bring `bytes` (a multiple of 16) of global memory at src (16-byte aligned) into L2 ahead of
// use; no completion to wait for.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Brings the L2 line holding address src into L2 (any alignment; no data reaches the thread).
__device__ __forceinline__ void prefetch_l2_line(const void* src) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(src));
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n"
        " .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait for phase `parity` of `bar`. Returns false if it did not complete within
// `max_polls` polls (each try_wait may itself suspend the thread for a short while).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint32_t max_polls) {
    for (uint32_t i = 0; i < max_polls; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

}  // namespace dev
}  // namespace gdn
