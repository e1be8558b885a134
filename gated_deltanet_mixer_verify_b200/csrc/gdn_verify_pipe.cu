// gdn_verify_pipe.cu -- persistent, warp-specialised form of the tensor-core verify mixer for
// d_k = d_v = 128, 2 <= T <= 8, with the commit fused at device accept counts.
//
// The block form is that of gdn_verify_tc.cu: the 2T dots per state row P = S_0 [Khat; Qhat]^T
// on tcgen05 (kind::tf32, three passes S_hi B_hi + S_hi B_lo + S_lo B_hi), the T x T algebra on
// the CUDA cores. Here the write vectors u = (I + A)^-1 x are formed per state row, so that
//   o_t = d_t r_t + sum_{m<=t} Cq[t][m] u_m   and   S_L = d_{L-1} S_0 + sum_{t<L} c_t u_t khat_t^T
// (c_t = e^{G_{L-1} - G_t}): the same sums as the folded coefficients Mo = Cq Tm and commit keys
// Keff_s = sum_t c_t Tm[t][s] khat_t, associated the other way. One CTA per SM walks its
// (sequence, value head) items, and every stage of a head has warps of its own, so that the
// stages of consecutive heads overlap:
//   - producer (warp 12, one thread): the state tile of head j by TMA into one of two 64 KB
//     buffers, as soon as the main group has read head j - 2's tile for its commit; an L2
//     prefetch of the next head's tile, so that the TMA reads it from L2;
//   - loader (warp 14): head j's q, k, v rows by bulk copies, and its gates (decays, beta, the
//     commit decays at its accept count) from the gate inputs, into one of two staging buffers,
//     one head ahead of the prep group;
//   - prep group (warps 0..3): head j's normalised keys and queries (the MMA's B operand, split
//     into tf32 high and low parts, and the keys in fp32), the Gram matrix, the decayed
//     coefficients A and Cq and (I + A)^-1, into one of two operand buffers;
//   - MMA issuer (warp 13, one thread): for head j, the two passes over the shared-memory tile
//     as soon as it and the operands are there, then the third pass (A = S_lo from tensor
//     memory) one 32-column block at a time, as the main group splits the tile;
//   - main group (warps 4..11): per head, the dots from tensor memory, x_s, u_t and the outputs;
//     then the split S_lo = S - trunc_tf32(S) of the next head's tile into tensor memory, block
//     by block (whose third pass then overlaps the rest); then this head's committed rows
//     (coalesced 512-byte rows, streaming stores).
//
// Every wait is bounded. Each thread of a group waits for itself, and the group then ORs its
// failures (and the CTA's abort flag) in a named barrier, so that all its threads take the same
// branch; a wait that runs out sets GDN_STATUS_WAIT_TIMEOUT and an abort flag that every other
// role's waits check, the CTA stops writing, drains its copies and MMAs (bounded) and frees its
// tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cstddef>

#include "gdn_device.cuh"
#include "gdn_internal.cuh"
#include "gdn_tc.cuh"

namespace gdn {
namespace {
using namespace dev;

constexpr int DK = 128;
constexpr int DV = 128;
constexpr int TM = 8;                    // block length bound (N = 2 TM = 16)
constexpr int NB = 2 * TM;               // rows of the B operand: khat_0..7, qhat_0..7
constexpr int kPrep = 128;               // warps 0..3
constexpr int kMain = 256;               // warps 4..11
constexpr int kProducerWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kLoaderWarp = 14;
constexpr int kThreads = 480;
constexpr int kBarPrep = 1;              // named barriers
constexpr int kBarMain = 2;
constexpr uint32_t kTileBytes = DV * DK * 4;
constexpr uint32_t kMaxPolls = 1u << 24;
constexpr uint32_t kTmemCols = 256;      // S_lo at 0..127, the dots of two heads at 128..191
constexpr uint32_t kDots = 128;

// One head's operands, written by the prep group (from the loader's gates) and read by the main
// group; arrays read with 16-byte accesses are 16-byte aligned.
struct HeadCtx {
    float K[TM][DK];                 // khat_t in fp32 (zero past T): commit keys
    float V[TM][DV];                 // v_t in fp32 (zero past T)
    alignas(16) float Tm[TM][TM];    // (I + A)^-1, unit lower triangular
    alignas(16) float Cq[TM][TM];    // e^{G_t - G_s} qhat_t . khat_s (s <= t < T)
    alignas(16) float D[TM];         // e^{G_t} (zero past T)
    alignas(16) float Beta[TM];      // sigmoid(b_t) (zero past T)
    alignas(16) float Ec[TM];        // e^{G_{L-1} - G_t} for t < L, else zero
    float DL;                        // e^{G_{L-1}} (1 for L <= 0)
    int L;                           // accept count; -1: out of range (nothing committed)
    int pad[2];
};

// A head's k, q and v rows (T each) as copied from global memory, in the input type: row t
// k_t, row TM + t q_t, row 2 TM + t v_t (rows past T are not written). Rows are 576 bytes
// apart (room for fp32 rows, and two bf16 rows' 64-byte spans fall in different banks).
constexpr uint32_t kStageRowBytes = DK * 4 + 64;

struct StageGates {                  // the loader's gates of one head
    alignas(16) float G[TM];         // inclusive prefix sums of the log-decays
    alignas(16) float D[TM];
    alignas(16) float Beta[TM];
    alignas(16) float Ec[TM];
    float DL;
    int L;
    int pad[2];
};

struct __align__(1024) PipeSmem {
    float S[2][DV * DK];             // state tiles, SW128 K-major (4 blocks of [128 rows][32])
    float B2[2][2 * NB * DK];        // [khat; qhat] high parts (rows 0..15), low parts (16..31), SW128
    HeadCtx ctx[2];
    alignas(16) unsigned char in[2][3 * TM][kStageRowBytes];   // loader -> prep staging
    StageGates gates[2];
    // prep group scratch
    alignas(16) float Gram[NB][TM];
    alignas(16) float G[TM];
    alignas(16) float A[TM][TM];
    // main group scratch
    alignas(16) float X[DV][TM];     // c_t u_t per state row: the commit's coefficients
    int abort;                       // a bounded wait ran out somewhere in the CTA
    uint32_t tmem;
    uint64_t full[2];                // state tile landed (TMA)
    uint64_t ctx_full[2];            // operands of a head ready (prep group)
    uint64_t ctx_empty[2];           // main group done with a head's operands
    uint64_t committed[2];           // the main group has read S[i] for its commit (buffer free)
    uint64_t mma_done[2];            // a head's dots in tensor memory
    uint64_t split_done[4];          // 32-column block kb of the next head's S_lo in tensor memory
    uint64_t in_full[2];             // a head's rows and gates staged (loader)
    uint64_t in_empty[2];            // the prep group has read a head's staged inputs
};

static_assert(sizeof(PipeSmem) <= 227 * 1024, "shared memory of one CTA");
static_assert(offsetof(PipeSmem, B2) % 1024 == 0 && offsetof(PipeSmem, ctx) % 16 == 0 &&
                  offsetof(PipeSmem, in) % 16 == 0 && offsetof(PipeSmem, gates) % 16 == 0 &&
                  offsetof(PipeSmem, A) % 16 == 0 && offsetof(PipeSmem, X) % 16 == 0 &&
                  sizeof(HeadCtx) % 16 == 0 && sizeof(StageGates) % 16 == 0 && offsetof(HeadCtx, Tm) % 16 == 0 &&
                  offsetof(HeadCtx, Cq) % 16 == 0 && offsetof(HeadCtx, D) % 16 == 0 &&
                  offsetof(HeadCtx, Beta) % 16 == 0 && offsetof(HeadCtx, Ec) % 16 == 0,
              "16-byte accesses to shared memory need 16-byte aligned arrays");

__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void set_abort(PipeSmem& sm, const VerifyArgs& p) {
    if (atomicExch(&sm.abort, 1) == 0 && p.status_word) atomicOr(p.status_word, kStatusWaitTimeout);
}

// Bounded wait that also gives up once another role has aborted. One thread.
__device__ __forceinline__ bool wait_or_abort(PipeSmem& sm, const VerifyArgs& p, uint64_t* bar, uint32_t parity) {
    for (uint32_t i = 0; i < kMaxPolls; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 63u && *reinterpret_cast<volatile int*>(&sm.abort)) return false;
    }
    set_abort(sm, p);
    return false;
}

// Expect `bytes` more transaction bytes in the current phase of `bar`, without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Named barrier `id` over `nthreads` threads that also ORs `pred` across them: every thread
// gets the same answer, so a group takes the same branch after it.
__device__ __forceinline__ bool named_sync_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n"
        " .reg .pred p, q;\n"
        " setp.ne.u32 p, %1, 0;\n"
        " barrier.red.or.pred q, %2, %3, p;\n"
        " selp.u32 %0, 1, 0, q;\n"
        "}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ bool aborted(PipeSmem& sm) { return *reinterpret_cast<volatile int*>(&sm.abort) != 0; }

// Committed rows for LL accepted tokens to dst (global, the head's state): S_L = dl S_0 +
// sum_{t<LL} X[row][t] khat_t (X = c_t u_t; LL = 0: S_0 copied). One warp per 16 rows
// (row = w + 8 i), a lane per 16-byte chunk, so each row leaves as one coalesced 512-byte store.
template <int LL>
__device__ __forceinline__ void commit_rows(const float* S, float* dst, const HeadCtx& c, const float (*X)[TM],
                                            int w, int lane) {
    const int chunk = lane;   // columns 4 chunk .. +3
    const int kb = chunk >> 3, cc = chunk & 7;
    float4 ke[LL > 0 ? LL : 1];
#pragma unroll
    for (int t = 0; t < LL; ++t) ke[t] = *reinterpret_cast<const float4*>(&c.K[t][4 * chunk]);
    const float2 dl2 = make_float2(c.DL, c.DL);
#pragma unroll 4
    for (int i = 0; i < DV / 8; ++i) {
        const int row = w + 8 * i;
        const float4 sv = *reinterpret_cast<const float4*>(&S[(kb * DV * 128 + row * 128 + ((cc ^ (row & 7)) << 4)) / 4]);
        float2 r0 = make_float2(sv.x, sv.y), r1 = make_float2(sv.z, sv.w);
        if (LL > 0) {
            r0 = __fmul2_rn(r0, dl2);
            r1 = __fmul2_rn(r1, dl2);
            float xv[8];
            const float4 x0 = *reinterpret_cast<const float4*>(&X[row][0]);
            xv[0] = x0.x; xv[1] = x0.y; xv[2] = x0.z; xv[3] = x0.w;
            if (LL > 4) {
                const float4 x1 = *reinterpret_cast<const float4*>(&X[row][4]);
                xv[4] = x1.x; xv[5] = x1.y; xv[6] = x1.z; xv[7] = x1.w;
            }
#pragma unroll
            for (int t = 0; t < LL; ++t) {
                const float2 xs = make_float2(xv[t], xv[t]);
                r0 = __ffma2_rn(xs, make_float2(ke[t].x, ke[t].y), r0);
                r1 = __ffma2_rn(xs, make_float2(ke[t].z, ke[t].w), r1);
            }
        }
        __stcs(reinterpret_cast<float4*>(dst + (size_t)row * DK) + chunk, make_float4(r0.x, r0.y, r1.x, r1.y));
    }
}

// Eight floats of shared memory (16-byte aligned) into registers by two 16-byte loads.
__device__ __forceinline__ void unpack8(const float* src, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(src);
    const float4 b = *reinterpret_cast<const float4*>(src + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Four consecutive input elements of a staged shared-memory row, from element i (a multiple
// of 4): one 8-byte load for bf16, one 16-byte load for fp32.
template <typename T>
__device__ __forceinline__ void ld4_smem(const unsigned char* row, int i, float* x);
template <>
__device__ __forceinline__ void ld4_smem<float>(const unsigned char* row, int i, float* x) {
    const float4 a = *reinterpret_cast<const float4*>(row + 4 * i);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}
template <>
__device__ __forceinline__ void ld4_smem<__nv_bfloat16>(const unsigned char* row, int i, float* x) {
    const uint2 u = *reinterpret_cast<const uint2*>(row + 2 * i);
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xffff0000u);
}

// Main group: block kb (columns 32 kb .. +31) of S_lo = S - trunc_tf32(S) of tile S into tensor
// memory (columns 0..127 = K). Thread (row, half) takes 16 columns of its row, its warp's lanes.
__device__ __forceinline__ void split_block(const float* S, uint32_t tmem, int kb, int row, int half, int lane_base) {
    float v[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int ch = 4 * half + q;   // 16-byte chunk of the row's 128-byte segment in block kb
        const float4 xs = *reinterpret_cast<const float4*>(&S[(kb * DV * 128 + row * 128 + ((ch ^ (row & 7)) << 4)) / 4]);
        v[4 * q + 0] = xs.x - tc::tf32_hi(xs.x);
        v[4 * q + 1] = xs.y - tc::tf32_hi(xs.y);
        v[4 * q + 2] = xs.z - tc::tf32_hi(xs.z);
        v[4 * q + 3] = xs.w - tc::tf32_hi(xs.w);
    }
    tc::tmem_st16_nowait(tmem + ((uint32_t)lane_base << 16) + 32 * kb + 16 * half, v);
    tc::tmem_st_wait();
}

template <typename InT, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    gdn_verify_pipe_kernel(const __grid_constant__ CUtensorMap smap, const VerifyArgs p, int prefetch) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    PipeSmem& sm = *reinterpret_cast<PipeSmem*>(smem_raw);
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int T = p.T;
    const int nitems = p.B * p.Hv;
    const int G = gridDim.x;
    const int n = ((int)blockIdx.x < nitems) ? (nitems - 1 - (int)blockIdx.x) / G + 1 : 0;   // heads of this CTA
    auto item_of = [&](int j) { return (int)blockIdx.x + j * G; };
    const size_t tok_stride = (size_t)p.Hv * DV;   // between tokens in v and o

    if ((smem_u32(smem_raw) & 1023u) != 0) {   // the swizzled tiles need 1024-byte alignment
        if (tid == 0 && p.status_word) atomicOr(p.status_word, kStatusWaitTimeout);
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.ctx_full[i], 1);
            mbar_init(&sm.ctx_empty[i], 1);
            mbar_init(&sm.committed[i], 1);
            mbar_init(&sm.mma_done[i], 1);
            mbar_init(&sm.in_full[i], 1);
            mbar_init(&sm.in_empty[i], 1);
        }
        for (int kb = 0; kb < 4; ++kb) mbar_init(&sm.split_done[kb], 1);
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tc::tmem_alloc(&sm.tmem, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = sm.tmem;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            int loads = 0;   // tiles requested
            for (int j = 0; j < n; ++j) {
                const int buf = j & 1;
                // head j - 2's tile has been read for its commit
                if (j >= 2 && !wait_or_abort(sm, p, &sm.committed[buf], ((j - 2) >> 1) & 1)) break;
                mbar_arrive_expect_tx(&sm.full[buf], kTileBytes);
                for (int kb = 0; kb < 4; ++kb)
                    tc::tma_load_2d(&sm.S[buf][kb * DV * 32], &smap, kb * 32, item_of(j) * DV, &sm.full[buf]);
                ++loads;
                if (prefetch && j + 1 < n) bulk_prefetch_l2(p.state_in + (size_t)item_of(j + 1) * DV * DK, kTileBytes);
            }
            // On an abort, the tiles in flight land (bounded) before the CTA exits.
            if (*reinterpret_cast<volatile int*>(&sm.abort))
                for (int j = max(0, loads - 2); j < loads; ++j) mbar_wait_bounded(&sm.full[j & 1], (j >> 1) & 1, kMaxPolls);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id32 = tc::idesc_tf32(DV, 2 * NB), id16 = tc::idesc_tf32(DV, NB);
            int pending = -1;   // last head whose MMAs were issued and committed
            for (int j = 0; j < n; ++j) {
                const int buf = j & 1;
                const uint32_t ph = (j >> 1) & 1;
                if (!wait_or_abort(sm, p, &sm.full[buf], ph)) break;
                if (!wait_or_abort(sm, p, &sm.ctx_full[buf], ph)) break;
                tc::fence_after_sync();
                const uint32_t dots = tmem + kDots + 32 * buf;
                const uint32_t as = smem_u32(sm.S[buf]);
                const uint32_t bb = smem_u32(sm.B2[buf]);
                // Columns 0..15 accumulate S B_hi + S_lo B_hi, columns 16..31 S B_lo.
#pragma unroll
                for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        tc::mma_tf32_ss(dots, tc::desc_kmajor_sw128(as + kb * DV * 128 + ks * 32),
                                        tc::desc_kmajor_sw128(bb + kb * 2 * NB * 128 + ks * 32), id32, kb + ks > 0);
                // The third pass, block by block as the main group splits the tile.
                bool split_ok = true;
                for (int kb = 0; kb < 4 && split_ok; ++kb) {
                    split_ok = wait_or_abort(sm, p, &sm.split_done[kb], j & 1);
                    tc::fence_after_sync();
                    if (split_ok) {
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            tc::mma_tf32_ts(dots, tmem + kb * 32 + ks * 8,
                                            tc::desc_kmajor_sw128(bb + kb * 2 * NB * 128 + ks * 32), id16, true);
                    }
                }
                tc::mma_commit(&sm.mma_done[buf]);
                pending = j;
                if (!split_ok) break;
            }
            // The last committed MMAs finish before the tensor memory is freed (at once unless
            // the CTA aborted: the main group has waited for every head's).
            if (pending >= 0) mbar_wait_bounded(&sm.mma_done[pending & 1], (pending >> 1) & 1, kMaxPolls);
        }
        __syncwarp();
    } else if (warp == kLoaderWarp) {
        // ------------------------------------------------------------------ loader
        // Head j's k, q, v rows by bulk copies (lane t: token t's three rows), and its gates,
        // into staging buffer j & 1 once the prep group has read head j - 2's. The buffer's
        // phase completes when the copies have landed and lane 0 has arrived after the gates
        // are stored.
        const size_t es = p.in_bf16 ? 2 : 4;
        const uint32_t row_bytes = (uint32_t)(DK * es);
        // The gate inputs of the next head are requested one iteration early (a plain load
        // waits behind the state traffic).
        float na = 0.f, nb = 0.f, nalog = 0.f, ndtb = 0.f;
        int nL = 0;
        auto load_gate_inputs = [&](int jj) {
            const int it = item_of(jj);
            const int hh = it % p.Hv, bb = it / p.Hv;
            if (lane < T) {
                const size_t gi = ((size_t)bb * T + lane) * p.Hv + hh;
                na = ld_in<InT>(p.a, gi);
                nb = ld_in<InT>(p.b, gi);
            }
            nalog = p.A_log[hh];
            ndtb = p.dt_bias[hh];
            nL = p.accept_len[bb];
        };
        if (n > 0) load_gate_inputs(0);
        int issued = 0;
        for (int j = 0; j < n; ++j) {
            const int buf = j & 1;
            bool ok = true;
            if (j >= 2) {
                if (lane == 0) ok = wait_or_abort(sm, p, &sm.in_empty[buf], ((j - 2) >> 1) & 1);
                ok = __shfl_sync(kFull, ok, 0);
            }
            if (!ok) break;
            const int it = item_of(j);
            const int hh = it % p.Hv, bb = it / p.Hv, gg = hh / (p.Hv / p.Hk);
            uint64_t* bar = &sm.in_full[buf];
            if (lane == 0) mbar_expect_tx(bar, 3u * T * row_bytes);
            __syncwarp();
            if (lane < T) {
                const char* kq = static_cast<const char*>(p.k) + (((size_t)bb * T + lane) * p.Hk + gg) * DK * es;
                const char* qq = static_cast<const char*>(p.q) + (((size_t)bb * T + lane) * p.Hk + gg) * DK * es;
                const char* vq = static_cast<const char*>(p.v) + (((size_t)bb * T + lane) * p.Hv + hh) * DV * es;
                bulk_g2s(sm.in[buf][lane], kq, row_bytes, bar);
                bulk_g2s(sm.in[buf][TM + lane], qq, row_bytes, bar);
                bulk_g2s(sm.in[buf][2 * TM + lane], vq, row_bytes, bar);
            }
            const float a_in = na, b_in = nb, alog = nalog, dtb = ndtb;
            const int L_in = nL;
            if (j + 1 < n) load_gate_inputs(j + 1);
            // Gates (lane t = token t): g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b),
            // the inclusive prefix sum G of g, d = e^G, and the commit decays at the accept count.
            float gl = 0.f, be = 0.f;
            if (lane < T) {
                gl = -expf(alog) * softplus_f(a_in + dtb);
                be = 1.f / (1.f + expf(-b_in));
            }
            float Gs = gl;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float yy = __shfl_up_sync(kFull, Gs, off);
                if (lane >= off) Gs += yy;
            }
            int L = L_in;
            if (L < 0 || L > T) {
                if (lane == 0 && p.status_word && hh == 0) atomicOr(p.status_word, kStatusBadAccept);
                L = -1;
            }
            const float D = (lane < T) ? expf(Gs) : 0.f;
            const float Glast = __shfl_sync(kFull, Gs, L > 0 ? L - 1 : 0);
            const float DL = __shfl_sync(kFull, D, L > 0 ? L - 1 : 0);
            StageGates& gs = sm.gates[buf];
            if (lane < TM) {
                gs.G[lane] = Gs;
                gs.D[lane] = D;
                gs.Beta[lane] = be;
                gs.Ec[lane] = (L > 0 && lane < L) ? expf(Glast - Gs) : 0.f;
            }
            if (lane == 0) {
                gs.DL = (L > 0) ? DL : 1.f;
                gs.L = L;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
            ++issued;
        }
        // On an abort, the copies in flight land (bounded) before the CTA exits.
        if (lane == 0 && *reinterpret_cast<volatile int*>(&sm.abort))
            for (int j = max(0, issued - 2); j < issued; ++j) mbar_wait_bounded(&sm.in_full[j & 1], (j >> 1) & 1, kMaxPolls);
        __syncwarp();
    } else if (warp < 4) {
        // ------------------------------------------------------------------ prep group
        const int c8 = tid & 7;            // columns 32 m + 4 c8 .. +3 (m = 0..3) of one vector
        const int nrow = tid >> 3;         // 0..15 = NB rows: khat_0..7, qhat_0..7
        const bool isq = nrow >= TM;
        const int tq = isq ? nrow - TM : nrow;
        const bool live = tq < T;
        for (int j = 0; j < n; ++j) {
            const int buf = j & 1;
            bool ok = wait_or_abort(sm, p, &sm.in_full[buf], (j >> 1) & 1);
            if (ok && j >= 2) ok = wait_or_abort(sm, p, &sm.ctx_empty[buf], ((j - 2) >> 1) & 1);
            if (named_sync_or(kBarPrep, kPrep, !ok || aborted(sm))) break;
            HeadCtx& c = sm.ctx[buf];
            const StageGates& gs = sm.gates[buf];
            float x[16];
            if (live) {
                const unsigned char* src = sm.in[buf][isq ? TM + tq : tq];
#pragma unroll
                for (int m = 0; m < 4; ++m) ld4_smem<InT>(src, 32 * m + 4 * c8, &x[4 * m]);
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) x[e] = 0.f;
            }
            // Normalised khat_t, qhat_t: the split B tiles of the MMA, and the keys in fp32.
            {
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < 16; ++e) ss = fmaf(x[e], x[e], ss);
                ss = group_sum<8>(ss);
                const float inv = live ? (isq ? p.scale : 1.f) / sqrtf(ss + p.l2_eps) : 0.f;
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    const int col = 32 * qd + 4 * c8;
                    float4 y, hi, lo;
                    y = make_float4(x[4 * qd] * inv, x[4 * qd + 1] * inv, x[4 * qd + 2] * inv, x[4 * qd + 3] * inv);
                    x[4 * qd] = y.x;
                    x[4 * qd + 1] = y.y;
                    x[4 * qd + 2] = y.z;
                    x[4 * qd + 3] = y.w;
                    hi = make_float4(tc::tf32_hi(y.x), tc::tf32_hi(y.y), tc::tf32_hi(y.z), tc::tf32_hi(y.w));
                    lo = make_float4(y.x - hi.x, y.y - hi.y, y.z - hi.z, y.w - hi.w);
                    *reinterpret_cast<float4*>(&sm.B2[buf][tc::sw128_offset(nrow, col, 2 * NB) / 4]) = hi;
                    *reinterpret_cast<float4*>(&sm.B2[buf][tc::sw128_offset(NB + nrow, col, 2 * NB) / 4]) = lo;
                    if (!isq) *reinterpret_cast<float4*>(&c.K[nrow][col]) = y;
                }
            }
            tc::fence_proxy_async_smem();   // the tensor core reads the B tiles written above
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                const unsigned char* vr = sm.in[buf][2 * TM + t];
                c.V[t][tid] = (t < T) ? (p.in_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(vr)[tid])
                                                   : reinterpret_cast<const float*>(vr)[tid])
                                      : 0.f;
            }
            if (tid < TM) {
                sm.G[tid] = gs.G[tid];
                c.D[tid] = gs.D[tid];
                c.Beta[tid] = gs.Beta[tid];
                c.Ec[tid] = gs.Ec[tid];
            }
            if (tid == 0) {
                c.DL = gs.DL;
                c.L = gs.L;
            }
            named_sync(kBarPrep, kPrep);
            if (tid == 0) mbar_arrive(&sm.in_empty[buf]);   // the staged inputs have been read
            // Gram rows [Khat; Qhat] Khat^T: thread (row n, lane c8) dots its 16 normalised
            // columns with those of each khat_s; the row's 8 lanes reduce them.
            {
                float part[TM];
#pragma unroll
                for (int s = 0; s < TM; ++s) {
                    float d = 0.f;
#pragma unroll
                    for (int qd = 0; qd < 4; ++qd) {
                        const float4 kk = *reinterpret_cast<const float4*>(&c.K[s][32 * qd + 4 * c8]);
                        d = fmaf(x[4 * qd], kk.x, d);
                        d = fmaf(x[4 * qd + 1], kk.y, d);
                        d = fmaf(x[4 * qd + 2], kk.z, d);
                        d = fmaf(x[4 * qd + 3], kk.w, d);
                    }
                    part[s] = d;
                }
                Halve<TM, 4>::run(part, c8);
                sm.Gram[nrow][c8] = part[0];
            }
            named_sync(kBarPrep, kPrep);
            // The decayed coefficients, one entry per thread ...
            if (tid < TM * TM) {
                const int t = tid / TM, s = tid % TM;
                const bool inq = t < T && s <= t;
                const float dec = inq ? expf(sm.G[t] - sm.G[s]) : 0.f;
                sm.A[t][s] = (inq && s < t) ? c.Beta[t] * dec * sm.Gram[t][s] : 0.f;
                c.Cq[t][s] = inq ? dec * sm.Gram[TM + t][s] : 0.f;
            }
            named_sync(kBarPrep, kPrep);
            // ... and the unit-triangular inverse Tm = (I + A)^-1 by forward substitution (warp 0,
            // lane s = column s); then one arrival for the group.
            if (warp == 0) {
                if (lane < TM) {
                    const int s = lane;
                    float a[TM][TM];
#pragma unroll
                    for (int t = 0; t < TM; ++t) unpack8(sm.A[t], a[t]);
                    float col[TM];
#pragma unroll
                    for (int t = 0; t < TM; ++t) {
                        float xx = (t == s) ? 1.f : 0.f;
#pragma unroll
                        for (int m = 0; m < t; ++m) xx = fmaf(-a[t][m], col[m], xx);
                        col[t] = (t >= s) ? xx : 0.f;
                        c.Tm[t][s] = col[t];
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.ctx_full[buf]);
            }
        }
    } else {
        // ------------------------------------------------------------------ main group
        const int gt = tid - kPrep;        // 0..255
        const int gw = gt >> 5;            // 0..7
        const int row = gt & (DV - 1);     // the thread's tensor-memory lane (= state row)
        const int half = gt >> 7;
        const int lane_base = 32 * (warp & 3);
        const bool leader = gt == 0;
        const bool in_place = p.state_out == p.state_in;
        OutT* op = reinterpret_cast<OutT*>(p.o);
        // S_lo of head i's tile (buffer i & 1), block by block, each block announced to the MMA
        // issuer as soon as every thread has stored its part.
        auto split = [&](int i) -> bool {
            const bool ok = wait_or_abort(sm, p, &sm.full[i & 1], (i >> 1) & 1);
            if (named_sync_or(kBarMain, kMain, !ok || aborted(sm))) return false;
#pragma unroll 1
            for (int kb = 0; kb < 4; ++kb) {
                split_block(sm.S[i & 1], tmem, kb, row, half, lane_base);
                tc::fence_before_sync();
                named_sync(kBarMain, kMain);
                if (leader) mbar_arrive(&sm.split_done[kb]);
            }
            return true;
        };
        bool ok = n > 0 && split(0);
        for (int i = 0; i < n && ok; ++i) {
            const int buf = i & 1;
            const uint32_t ph = (i >> 1) & 1;
            const int item = item_of(i);
            const int h = item % p.Hv;
            const int b = item / p.Hv;
            const size_t vo_base = ((size_t)b * T * p.Hv + h) * DV;
            bool ok_t = wait_or_abort(sm, p, &sm.ctx_full[buf], ph);
            if (ok_t) ok_t = wait_or_abort(sm, p, &sm.mma_done[buf], ph);
            if (named_sync_or(kBarMain, kMain, !ok_t || aborted(sm))) break;
            tc::fence_after_sync();
            const HeadCtx& c = sm.ctx[buf];
            // Dots from tensor memory; x_s, the write vectors u_t = sum_{s<=t} Tm[t][s] x_s, and
            // the outputs of tokens 4 half .. +3.
            {
                float dots[16], dlo[16];
                const uint32_t dt = tmem + ((uint32_t)lane_base << 16) + kDots + 32 * buf;
                tc::tmem_ld16x2(dt, dt + 16, dots, dlo);
#pragma unroll
                for (int e = 0; e < 16; ++e) dots[e] += dlo[e];
                float be[TM], dd[TM], xs[TM], u[TM];
                unpack8(c.Beta, be);
                unpack8(c.D, dd);
#pragma unroll
                for (int s = 0; s < TM; ++s) xs[s] = be[s] * (c.V[s][row] - dd[s] * dots[s]);
#pragma unroll
                for (int t = 0; t < TM; ++t) {
                    float tm[TM];
                    unpack8(c.Tm[t], tm);
                    float acc = 0.f;
#pragma unroll
                    for (int s = 0; s <= t; ++s) acc = fmaf(tm[s], xs[s], acc);
                    u[t] = acc;
                }
                if (half == 0) {
                    float ec[TM];
                    unpack8(c.Ec, ec);
                    *reinterpret_cast<float4*>(&sm.X[row][0]) = make_float4(ec[0] * u[0], ec[1] * u[1], ec[2] * u[2], ec[3] * u[3]);
                    *reinterpret_cast<float4*>(&sm.X[row][4]) = make_float4(ec[4] * u[4], ec[5] * u[5], ec[6] * u[6], ec[7] * u[7]);
                }
#pragma unroll
                for (int tt = 0; tt < TM / 2; ++tt) {
                    const int t = (TM / 2) * half + tt;
                    if (t < T) {
                        float cq[TM];
                        unpack8(c.Cq[t], cq);
                        float ov = half ? dd[TM / 2 + tt] * dots[TM + TM / 2 + tt] : dd[tt] * dots[TM + tt];   // static indices
#pragma unroll
                        for (int m = 0; m < TM; ++m)
                            if (m <= t) ov = fmaf(cq[m], u[m], ov);
                        st_out<OutT>(op, vo_base + t * tok_stride + row, ov);
                    }
                }
            }
            tc::fence_before_sync();
            named_sync(kBarMain, kMain);   // X complete; this head's dots read
            // The next head's split (its tile in the other buffer): its third pass then runs on
            // the tensor cores while this head's commit stores.
            if (i + 1 < n && !split(i + 1)) break;
            // Commit at L (rollback / bad L: the initial state, written only out of place).
            const int L = c.L;
            const float* S = sm.S[buf];
            if (L > 0 || !in_place) {
                float* dst = p.state_out + (size_t)item * DV * DK;
                switch (L > 0 ? L : 0) {
                    case 1: commit_rows<1>(S, dst, c, sm.X, gw, lane); break;
                    case 2: commit_rows<2>(S, dst, c, sm.X, gw, lane); break;
                    case 3: commit_rows<3>(S, dst, c, sm.X, gw, lane); break;
                    case 4: commit_rows<4>(S, dst, c, sm.X, gw, lane); break;
                    case 5: commit_rows<5>(S, dst, c, sm.X, gw, lane); break;
                    case 6: commit_rows<6>(S, dst, c, sm.X, gw, lane); break;
                    case 7: commit_rows<7>(S, dst, c, sm.X, gw, lane); break;
                    case 8: commit_rows<8>(S, dst, c, sm.X, gw, lane); break;
                    default: commit_rows<0>(S, dst, c, sm.X, gw, lane); break;
                }
            }
            named_sync(kBarMain, kMain);   // S[buf] and the head's operands are no longer read
            if (leader) {
                mbar_arrive(&sm.committed[buf]);
                mbar_arrive(&sm.ctx_empty[buf]);
            }
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == kMmaWarp) tc::tmem_dealloc(tmem, kTmemCols);
}

template <typename InT, typename OutT>
cudaError_t launch_pipe_t(const VerifyArgs& a, cudaStream_t stream) {
    constexpr size_t smem = sizeof(PipeSmem);
    cudaError_t e = ensure_smem_attr<gdn_verify_pipe_kernel<InT, OutT>>((int)smem);
    if (e != cudaSuccess) return e;
    CUtensorMap smap;
    e = tc::encode_tmap_f32_sw128(&smap, a.state_in, (uint64_t)a.B * a.Hv * DV, DK, DV);
    if (e != cudaSuccess) return e;
    int nsm = 0;
    e = current_sm_count(&nsm);
    if (e != cudaSuccess) return e;
    const int grid = std::min(a.B * a.Hv, nsm);
    gdn_verify_pipe_kernel<InT, OutT><<<grid, kThreads, smem, stream>>>(smap, a, 1);
    return cudaGetLastError();
}

}  // namespace

bool pipe_kernel_applies(const VerifyArgs& a, int num_sms) {
    return tc_kernel_applies(a, num_sms) && a.accept_len && a.state_out && !a.always_commit && !a.stash &&
           !a.prev_stash && !a.norm_z;
}

cudaError_t launch_verify_pipe(const VerifyArgs& a, cudaStream_t stream) {
    if (a.in_bf16)
        return a.out_bf16 ? launch_pipe_t<__nv_bfloat16, __nv_bfloat16>(a, stream)
                          : launch_pipe_t<__nv_bfloat16, float>(a, stream);
    return a.out_bf16 ? launch_pipe_t<float, __nv_bfloat16>(a, stream) : launch_pipe_t<float, float>(a, stream);
}

}  // namespace gdn
