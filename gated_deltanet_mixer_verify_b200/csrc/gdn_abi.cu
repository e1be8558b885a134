// gdn_abi.cu -- the extern "C" entry points of libgdn.so (declared in include/gdn.h):
// host-side argument checks, then one kernel launch on the caller's stream.
// No allocation, no host synchronisation, no copy of device data to the host.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "gdn.h"
#include "gdn_internal.cuh"
#include "gdn_prefill.cuh"

namespace {

thread_local char g_last_error[256] = "";

gdn_status fail(gdn_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return s;
}

gdn_status ok() {
    g_last_error[0] = '\0';
    return GDN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_dk(int dk) { return dk == 16 || dk == 32 || dk == 64 || dk == 128; }

// Checks common to every call. max_T: largest block length this call supports.
gdn_status check_shape(const gdn_shape* s, int max_T, const char* who) {
    if (!s) return fail(GDN_ERR_INVALID_ARG, "%s: shape is NULL", who);
    if (s->B < 0 || s->T < 1 || s->H_k < 1 || s->H_v < 1 || s->d_k < 1 || s->d_v < 1)
        return fail(GDN_ERR_INVALID_ARG, "%s: sizes must be positive (B may be 0)", who);
    if (s->H_v % s->H_k != 0)
        return fail(GDN_ERR_INVALID_ARG, "%s: H_v (%d) is not a multiple of H_k (%d)", who, s->H_v, s->H_k);
    if (s->in_dtype != GDN_F32 && s->in_dtype != GDN_BF16)
        return fail(GDN_ERR_INVALID_ARG, "%s: in_dtype %d unknown", who, s->in_dtype);
    if (s->out_dtype != GDN_F32 && s->out_dtype != GDN_BF16)
        return fail(GDN_ERR_INVALID_ARG, "%s: out_dtype %d unknown", who, s->out_dtype);
    if (!(s->l2_eps >= 0.f) || !(s->scale == s->scale))
        return fail(GDN_ERR_INVALID_ARG, "%s: l2_eps must be >= 0 and scale a number", who);
    if (s->B > 65535 || s->H_v > 65535 || (int64_t)s->B * s->H_v > (1 << 24))
        return fail(GDN_ERR_UNSUPPORTED, "%s: B, H_v <= 65535 and B * H_v <= 2^24 required", who);
    if (!supported_dk(s->d_k))
        return fail(GDN_ERR_UNSUPPORTED, "%s: d_k %d not built (16, 32, 64, 128)", who, s->d_k);
    if (s->d_v > 4096) return fail(GDN_ERR_UNSUPPORTED, "%s: d_v %d > 4096", who, s->d_v);
    if (s->T > max_T) return fail(GDN_ERR_UNSUPPORTED, "%s: T %d > %d", who, s->T, max_T);
    if (s->status_word && !aligned16(s->status_word) &&
        (reinterpret_cast<uintptr_t>(s->status_word) & 3u) != 0)
        return fail(GDN_ERR_INVALID_ARG, "%s: status_word misaligned", who);
    if (s->launch_flags & ~GDN_LAUNCH_PDL)
        return fail(GDN_ERR_INVALID_ARG, "%s: launch_flags 0x%x has unknown bits", who, s->launch_flags);
    return GDN_OK;
}

#define REQUIRE_PTR(p, who)                                                                   \
    do {                                                                                      \
        if (!(p)) return fail(GDN_ERR_INVALID_ARG, "%s: %s is NULL", who, #p);                \
        if (!aligned16(p)) return fail(GDN_ERR_INVALID_ARG, "%s: %s not 16-byte aligned", who, #p); \
    } while (0)

size_t state_bytes(const gdn_shape* s) {
    return (size_t)s->B * s->H_v * s->d_v * s->d_k * sizeof(float);
}

// Distinct or identical, never partially overlapping.
bool overlap_ok(const void* x, const void* y, size_t bytes) {
    if (x == y) return true;
    const char* a = static_cast<const char*>(x);
    const char* b = static_cast<const char*>(y);
    return a + bytes <= b || b + bytes <= a;
}

gdn::VerifyArgs make_args(const gdn_shape* s, const void* q, const void* k, const void* v,
                          const void* a, const void* b, const float* A_log, const float* dt_bias) {
    gdn::VerifyArgs x;
    memset(&x, 0, sizeof(x));
    x.B = s->B;
    x.T = s->T;
    x.Hk = s->H_k;
    x.Hv = s->H_v;
    x.dk = s->d_k;
    x.dv = s->d_v;
    x.in_bf16 = s->in_dtype == GDN_BF16;
    x.out_bf16 = s->out_dtype == GDN_BF16;
    x.q = q;
    x.k = k;
    x.v = v;
    x.a = a;
    x.b = b;
    x.A_log = A_log;
    x.dt_bias = dt_bias;
    x.l2_eps = s->l2_eps;
    x.scale = s->scale;
    x.status_word = s->status_word;
    x.pdl = (s->launch_flags & GDN_LAUNCH_PDL) != 0;
    return x;
}

gdn_status launched(cudaError_t e, const char* who) {
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "%s: launch failed: %s", who, cudaGetErrorString(e));
    return ok();
}

}  // namespace

namespace {

// gdn_verify_step and gdn_verify_step_gated (norm_z non-NULL: gated norm of the outputs).
gdn_status verify_impl(const char* who, const gdn_shape* shape, const void* q, const void* k, const void* v,
                       const void* a, const void* b, const float* A_log, const float* dt_bias,
                       const float* state_in, float* state_out, const int32_t* accept_len, const void* norm_z,
                       const float* norm_w, float norm_eps, void* o, float* stash, void* stream) {
    gdn_status st = check_shape(shape, 16, who);
    if (st != GDN_OK) return st;
    if (norm_z && shape->d_v % 4 != 0)
        return fail(GDN_ERR_UNSUPPORTED, "%s: the gated norm needs d_v a multiple of 4", who);
    if (norm_z && !(norm_eps >= 0.f)) return fail(GDN_ERR_INVALID_ARG, "%s: norm_eps must be >= 0", who);
    if (shape->B == 0) return ok();
    REQUIRE_PTR(q, who);
    REQUIRE_PTR(k, who);
    REQUIRE_PTR(v, who);
    REQUIRE_PTR(a, who);
    REQUIRE_PTR(b, who);
    REQUIRE_PTR(A_log, who);
    REQUIRE_PTR(dt_bias, who);
    REQUIRE_PTR(state_in, who);
    REQUIRE_PTR(o, who);
    if (norm_z) {
        REQUIRE_PTR(norm_z, who);
        REQUIRE_PTR(norm_w, who);
    }
    if (accept_len) {
        REQUIRE_PTR(accept_len, who);
        REQUIRE_PTR(state_out, who);
        if (!overlap_ok(state_in, state_out, state_bytes(shape)))
            return fail(GDN_ERR_INVALID_ARG, "%s: state_out partially overlaps state_in", who);
    } else if (!stash) {
        return fail(GDN_ERR_INVALID_ARG, "%s: stash is required when accept_len is NULL", who);
    }
    if (stash) REQUIRE_PTR(stash, who);
    gdn::VerifyArgs x = make_args(shape, q, k, v, a, b, A_log, dt_bias);
    x.state_in = state_in;
    x.state_out = accept_len ? state_out : nullptr;
    x.accept_len = accept_len;
    x.o = o;
    x.stash = stash;
    x.always_commit = 0;
    x.norm_z = norm_z;
    x.norm_w = norm_w;
    x.norm_eps = norm_eps;
    return launched(gdn::launch_verify(x, static_cast<cudaStream_t>(stream)), who);
}

}  // namespace

extern "C" {


gdn_status gdn_verify_step(const gdn_shape* shape, const void* q, const void* k, const void* v,
                           const void* a, const void* b, const float* A_log, const float* dt_bias,
                           const float* state_in, float* state_out, const int32_t* accept_len,
                           void* o, float* stash, void* stream) {
    return verify_impl("gdn_verify_step", shape, q, k, v, a, b, A_log, dt_bias, state_in, state_out, accept_len,
                       nullptr, nullptr, 0.f, o, stash, stream);
}

gdn_status gdn_verify_step_gated(const gdn_shape* shape, const void* q, const void* k, const void* v,
                                 const void* a, const void* b, const float* A_log, const float* dt_bias,
                                 const float* state_in, float* state_out, const int32_t* accept_len,
                                 const void* norm_z, const float* norm_w, float norm_eps, void* o, float* stash,
                                 void* stream) {
    const char* who = "gdn_verify_step_gated";
    if (!norm_z) return fail(GDN_ERR_INVALID_ARG, "%s: norm_z is NULL", who);
    return verify_impl(who, shape, q, k, v, a, b, A_log, dt_bias, state_in, state_out, accept_len, norm_z, norm_w,
                       norm_eps, o, stash, stream);
}

gdn_status gdn_gated_rmsnorm(int64_t rows, int32_t d, const void* x, int32_t x_dtype, const void* z,
                             int32_t z_dtype, const float* w, float eps, void* y, int32_t y_dtype, void* stream) {
    const char* who = "gdn_gated_rmsnorm";
    if (rows < 0 || d < 4 || d % 4 != 0 || d > 4096)
        return fail(GDN_ERR_INVALID_ARG, "%s: rows >= 0 and d a multiple of 4 in 4..4096 required", who);
    for (int32_t t : {x_dtype, z_dtype, y_dtype})
        if (t != GDN_F32 && t != GDN_BF16) return fail(GDN_ERR_INVALID_ARG, "%s: dtype %d unknown", who, t);
    if (!(eps >= 0.f)) return fail(GDN_ERR_INVALID_ARG, "%s: eps must be >= 0", who);
    if (rows > ((int64_t)1 << 33)) return fail(GDN_ERR_UNSUPPORTED, "%s: more than 2^33 rows", who);
    if (rows == 0) return ok();
    REQUIRE_PTR(x, who);
    REQUIRE_PTR(z, who);
    REQUIRE_PTR(w, who);
    REQUIRE_PTR(y, who);
    const size_t xb = (size_t)rows * d * (x_dtype == GDN_BF16 ? 2 : 4);
    const size_t yb = (size_t)rows * d * (y_dtype == GDN_BF16 ? 2 : 4);
    if (x != y) {
        const char* xp = static_cast<const char*>(x);
        const char* yp = static_cast<const char*>(y);
        if (xp < yp + yb && yp < xp + xb)
            return fail(GDN_ERR_INVALID_ARG, "%s: y partially overlaps x", who);
    } else if (x_dtype != y_dtype) {
        return fail(GDN_ERR_INVALID_ARG, "%s: in place needs x and y of one dtype", who);
    }
    gdn::NormArgs n;
    n.x = x;
    n.z = z;
    n.w = w;
    n.y = y;
    n.rows = rows;
    n.d = d;
    n.eps = eps;
    n.x_bf16 = x_dtype == GDN_BF16;
    n.z_bf16 = z_dtype == GDN_BF16;
    n.y_bf16 = y_dtype == GDN_BF16;
    return launched(gdn::launch_gated_rmsnorm(n, static_cast<cudaStream_t>(stream)), who);
}

gdn_status gdn_commit(const gdn_shape* shape, const float* state_in, float* state_out,
                      const float* stash, const int32_t* accept_len, void* stream) {
    const char* who = "gdn_commit";
    gdn_status st = check_shape(shape, 16, who);
    if (st != GDN_OK) return st;
    if (shape->B == 0) return ok();
    REQUIRE_PTR(state_in, who);
    REQUIRE_PTR(state_out, who);
    REQUIRE_PTR(stash, who);
    REQUIRE_PTR(accept_len, who);
    if (!overlap_ok(state_in, state_out, state_bytes(shape)))
        return fail(GDN_ERR_INVALID_ARG, "%s: state_out partially overlaps state_in", who);
    gdn::CommitArgs x;
    x.B = shape->B;
    x.T = shape->T;
    x.Hv = shape->H_v;
    x.dk = shape->d_k;
    x.dv = shape->d_v;
    x.state_in = state_in;
    x.state_out = state_out;
    x.stash = stash;
    x.accept_len = accept_len;
    x.status_word = shape->status_word;
    return launched(gdn::launch_commit(x, static_cast<cudaStream_t>(stream)), who);
}

gdn_status gdn_commit_and_verify(const gdn_shape* shape, int32_t prev_T, const void* q, const void* k,
                                 const void* v, const void* a, const void* b, const float* A_log,
                                 const float* dt_bias, float* state, const float* prev_stash,
                                 const int32_t* prev_accept_len, const int32_t* accept_len, void* o,
                                 float* stash, void* stream) {
    const char* who = "gdn_commit_and_verify";
    gdn_status st = check_shape(shape, 16, who);
    if (st != GDN_OK) return st;
    if (prev_T < 1 || prev_T > 16) return fail(GDN_ERR_INVALID_ARG, "%s: prev_T = %d not in 1..16", who, (int)prev_T);
    if (shape->B == 0) return ok();
    REQUIRE_PTR(q, who);
    REQUIRE_PTR(k, who);
    REQUIRE_PTR(v, who);
    REQUIRE_PTR(a, who);
    REQUIRE_PTR(b, who);
    REQUIRE_PTR(A_log, who);
    REQUIRE_PTR(dt_bias, who);
    REQUIRE_PTR(state, who);
    REQUIRE_PTR(prev_stash, who);
    REQUIRE_PTR(prev_accept_len, who);
    REQUIRE_PTR(o, who);
    if (accept_len) {
        REQUIRE_PTR(accept_len, who);
    } else if (!stash) {
        return fail(GDN_ERR_INVALID_ARG, "%s: stash is required when accept_len is NULL", who);
    }
    if (stash) REQUIRE_PTR(stash, who);
    gdn::VerifyArgs x = make_args(shape, q, k, v, a, b, A_log, dt_bias);
    x.state_in = state;
    x.state_out = state;
    x.accept_len = accept_len;
    x.o = o;
    x.stash = stash;
    x.always_commit = 0;
    cudaStream_t s0 = static_cast<cudaStream_t>(stream);
    int nsm = 0;
    cudaError_t e = gdn::current_sm_count(&nsm);
    if (e != cudaSuccess) return launched(e, who);
    if (gdn::tc_kernel_applies(x, nsm) && prev_T <= 8) {
        // One pass over the state: the tensor-core kernel applies the previous stash on-chip.
        x.prev_stash = prev_stash;
        x.prev_accept_len = prev_accept_len;
        x.prev_T = prev_T;
        return launched(gdn::launch_verify(x, s0), who);
    }
    // Other shapes: the previous commit in place, then the verify (an extra state pass).
    gdn::CommitArgs c;
    c.B = shape->B;
    c.T = prev_T;
    c.Hv = shape->H_v;
    c.dk = shape->d_k;
    c.dv = shape->d_v;
    c.state_in = state;
    c.state_out = state;
    c.stash = prev_stash;
    c.accept_len = prev_accept_len;
    c.status_word = shape->status_word;
    e = gdn::launch_commit(c, s0);
    if (e != cudaSuccess) return launched(e, who);
    if (!accept_len) x.state_out = nullptr;   // two-phase again: the state already holds the new base
    return launched(gdn::launch_verify(x, s0), who);
}

gdn_status gdn_decode_step(const gdn_shape* shape, const void* q, const void* k, const void* v,
                           const void* a, const void* b, const float* A_log, const float* dt_bias,
                           float* state, void* o, void* stream) {
    const char* who = "gdn_decode_step";
    gdn_status st = check_shape(shape, 1, who);
    if (st != GDN_OK) return st;
    if (shape->B == 0) return ok();
    REQUIRE_PTR(q, who);
    REQUIRE_PTR(k, who);
    REQUIRE_PTR(v, who);
    REQUIRE_PTR(a, who);
    REQUIRE_PTR(b, who);
    REQUIRE_PTR(A_log, who);
    REQUIRE_PTR(dt_bias, who);
    REQUIRE_PTR(state, who);
    REQUIRE_PTR(o, who);
    gdn::VerifyArgs x = make_args(shape, q, k, v, a, b, A_log, dt_bias);
    x.state_in = state;
    x.state_out = state;
    x.accept_len = nullptr;
    x.o = o;
    x.stash = nullptr;
    x.always_commit = 1;
    return launched(gdn::launch_verify(x, static_cast<cudaStream_t>(stream)), who);
}

size_t gdn_stash_bytes(const gdn_shape* shape) {
    if (check_shape(shape, 16, "gdn_stash_bytes") != GDN_OK) return 0;
    return (size_t)shape->B * shape->H_v *
           gdn::stash_floats_per_head(shape->T, shape->d_k, shape->d_v) * sizeof(float);
}

size_t gdn_chunk_prefill_workspace_bytes(const gdn_shape* shape, int32_t chunk) {
    if (gdn::check_prefill_shape(shape, chunk) != 0) return 0;
    return gdn::prefill_workspace_bytes(shape->B, shape->T, shape->H_k, shape->H_v, shape->d_k, shape->d_v, chunk);
}

int32_t gdn_chunk_prefill_pieces(int64_t T, int32_t chunk) {
    gdn_shape s{};
    s.B = 1;
    s.T = 1;
    s.H_k = 1;
    s.H_v = 1;
    s.d_k = 128;
    s.d_v = 128;
    if (T < 0 || gdn::check_prefill_shape(&s, chunk) != 0) return -1;
    return gdn::prefill_pieces((long long)T);
}

// Shape, chunk and workspace checks shared by the workspace-taking prefill entry points.
// Returns GDN_OK with *empty set when the batch is empty (nothing to launch).
static gdn_status prefill_checks(const gdn_shape* shape, int32_t chunk, const void* workspace, size_t workspace_bytes,
                                 const char* who, bool* empty) {
    *empty = false;
    if (!shape) return fail(GDN_ERR_INVALID_ARG, "%s: shape is NULL", who);
    gdn_status st = check_shape(shape, 1 << 30, who);
    if (st != GDN_OK) return st;
    if (gdn::check_prefill_shape(shape, chunk) != 0)
        return fail(GDN_ERR_UNSUPPORTED, "%s: only chunk 64 with d_k = d_v = 128 is built", who);
    if (shape->B == 0) {
        *empty = true;
        return ok();
    }
    const size_t need = gdn::prefill_workspace_bytes(shape->B, shape->T, shape->H_k, shape->H_v, shape->d_k,
                                                     shape->d_v, chunk);
    if (need > 0) {
        if (!workspace || workspace_bytes < need)
            return fail(GDN_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", who, need,
                        workspace_bytes);
        if (!aligned16(workspace)) return fail(GDN_ERR_INVALID_ARG, "%s: workspace not 16-byte aligned", who);
    }
    return GDN_OK;
}

gdn_status gdn_chunk_prefill(const gdn_shape* shape, int32_t chunk, const void* q, const void* k,
                             const void* v, const void* a, const void* b, const float* A_log,
                             const float* dt_bias, const float* state_in, float* state_out, void* o,
                             void* workspace, size_t workspace_bytes, void* stream) {
    const char* who = "gdn_chunk_prefill";
    bool empty = false;
    gdn_status st = prefill_checks(shape, chunk, workspace, workspace_bytes, who, &empty);
    if (st != GDN_OK || empty) return st;
    REQUIRE_PTR(q, who);
    REQUIRE_PTR(k, who);
    REQUIRE_PTR(v, who);
    REQUIRE_PTR(a, who);
    REQUIRE_PTR(b, who);
    REQUIRE_PTR(A_log, who);
    REQUIRE_PTR(dt_bias, who);
    REQUIRE_PTR(state_out, who);
    REQUIRE_PTR(o, who);
    if (state_in) {
        REQUIRE_PTR(state_in, who);
        if (!overlap_ok(state_in, state_out, state_bytes(shape)))
            return fail(GDN_ERR_INVALID_ARG, "%s: state_out partially overlaps state_in", who);
    }
    gdn::VerifyArgs x = make_args(shape, q, k, v, a, b, A_log, dt_bias);
    x.state_in = state_in;
    x.state_out = state_out;
    x.o = o;
    x.always_commit = 1;   // the state after the last prompt token is always written
    return launched(gdn::launch_prefill(x, chunk, workspace, workspace_bytes,
                                        static_cast<cudaStream_t>(stream)),
                    who);
}

gdn_status gdn_chunk_prefill_prepare(const gdn_shape* shape, int32_t chunk, const void* q, const void* k,
                                     const void* a, const void* b, const float* A_log, const float* dt_bias,
                                     void* workspace, size_t workspace_bytes, void* stream) {
    const char* who = "gdn_chunk_prefill_prepare";
    bool empty = false;
    gdn_status st = prefill_checks(shape, chunk, workspace, workspace_bytes, who, &empty);
    if (st != GDN_OK || empty) return st;
    REQUIRE_PTR(q, who);
    REQUIRE_PTR(k, who);
    REQUIRE_PTR(a, who);
    REQUIRE_PTR(b, who);
    REQUIRE_PTR(A_log, who);
    REQUIRE_PTR(dt_bias, who);
    gdn::VerifyArgs x = make_args(shape, q, k, nullptr, a, b, A_log, dt_bias);
    return launched(gdn::launch_prefill_prepare(x, workspace, static_cast<cudaStream_t>(stream)), who);
}

gdn_status gdn_chunk_prefill_scan(const gdn_shape* shape, int32_t chunk, const void* v, const float* state_in,
                                  float* state_out, void* o, void* workspace, size_t workspace_bytes,
                                  void* stream) {
    const char* who = "gdn_chunk_prefill_scan";
    bool empty = false;
    gdn_status st = prefill_checks(shape, chunk, workspace, workspace_bytes, who, &empty);
    if (st != GDN_OK || empty) return st;
    REQUIRE_PTR(v, who);
    REQUIRE_PTR(state_out, who);
    REQUIRE_PTR(o, who);
    if (state_in) {
        REQUIRE_PTR(state_in, who);
        if (!overlap_ok(state_in, state_out, state_bytes(shape)))
            return fail(GDN_ERR_INVALID_ARG, "%s: state_out partially overlaps state_in", who);
    }
    gdn::VerifyArgs x = make_args(shape, nullptr, nullptr, v, nullptr, nullptr, nullptr, nullptr);
    x.state_in = state_in;
    x.state_out = state_out;
    x.o = o;
    x.always_commit = 1;
    return launched(gdn::launch_prefill_scan(x, workspace, static_cast<cudaStream_t>(stream)), who);
}

gdn_status gdn_chunk_prefill_noalloc(const gdn_shape* shape, int32_t chunk, const void* q, const void* k,
                                     const void* v, const void* a, const void* b, const float* A_log,
                                     const float* dt_bias, const float* state_in, float* state_out, void* o,
                                     void* stream) {
    const char* who = "gdn_chunk_prefill_noalloc";
    if (!shape) return fail(GDN_ERR_INVALID_ARG, "%s: shape is NULL", who);
    gdn_status st = check_shape(shape, 1 << 30, who);
    if (st != GDN_OK) return st;
    if (gdn::check_prefill_shape(shape, chunk) != 0)
        return fail(GDN_ERR_UNSUPPORTED, "%s: only chunk 64 with d_k = d_v = 128 is built", who);
    if (shape->B == 0) return ok();
    const size_t need = gdn::prefill_workspace_bytes(shape->B, shape->T, shape->H_k, shape->H_v, shape->d_k,
                                                     shape->d_v, chunk);
    if (need > gdn::kNoAllocScratchBytes)
        return fail(GDN_ERR_UNSUPPORTED,
                    "%s: this shape needs %zu bytes of scratch, the fixed scratch holds %zu; "
                    "use gdn_chunk_prefill with a workspace",
                    who, need, gdn::kNoAllocScratchBytes);
    REQUIRE_PTR(q, who);
    REQUIRE_PTR(k, who);
    REQUIRE_PTR(v, who);
    REQUIRE_PTR(a, who);
    REQUIRE_PTR(b, who);
    REQUIRE_PTR(A_log, who);
    REQUIRE_PTR(dt_bias, who);
    REQUIRE_PTR(state_out, who);
    REQUIRE_PTR(o, who);
    if (state_in) {
        REQUIRE_PTR(state_in, who);
        if (!overlap_ok(state_in, state_out, state_bytes(shape)))
            return fail(GDN_ERR_INVALID_ARG, "%s: state_out partially overlaps state_in", who);
    }
    gdn::VerifyArgs x = make_args(shape, q, k, v, a, b, A_log, dt_bias);
    x.state_in = state_in;
    x.state_out = state_out;
    x.o = o;
    x.always_commit = 1;
    return launched(gdn::launch_prefill_noalloc(x, chunk, static_cast<cudaStream_t>(stream)), who);
}

const char* gdn_status_string(gdn_status status) {
    switch (status) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG: bad shape, NULL or misaligned pointer";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: size or type not built into this library";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA: a kernel launch failed";
        case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE: workspace missing or too small";
    }
    return "unknown gdn_status";
}

const char* gdn_last_error(void) { return g_last_error; }

gdn_status gdn_short_conv(const gdn_shape* shape, int32_t conv_k, const void* q, const void* k,
                          const void* v, const float* conv_w, const void* hist_in, void* hist_out,
                          const int32_t* accept_len, void* q_out, void* k_out, void* v_out, void* stream) {
    const char* who = "gdn_short_conv";
    gdn_status st = check_shape(shape, 1 << 20, who);
    if (st != GDN_OK) return st;
    if (conv_k < 2 || conv_k > 4) return fail(GDN_ERR_UNSUPPORTED, "%s: conv_k %d not built (2, 3, 4)", who, conv_k);
    if (shape->d_k % 8 != 0 || shape->d_v % 8 != 0)
        return fail(GDN_ERR_UNSUPPORTED, "%s: d_k and d_v must be multiples of 8", who);
    const bool outputs = q_out || k_out || v_out;
    if (outputs && !(q_out && k_out && v_out))
        return fail(GDN_ERR_INVALID_ARG, "%s: q_out, k_out, v_out must be all given or all NULL", who);
    if (!outputs && !hist_out) return fail(GDN_ERR_INVALID_ARG, "%s: nothing to write", who);
    if (shape->B == 0) return ok();
    REQUIRE_PTR(q, who);
    REQUIRE_PTR(k, who);
    REQUIRE_PTR(v, who);
    REQUIRE_PTR(hist_in, who);
    if (outputs) {
        REQUIRE_PTR(conv_w, who);
        REQUIRE_PTR(q_out, who);
        REQUIRE_PTR(k_out, who);
        REQUIRE_PTR(v_out, who);
    }
    if (hist_out) REQUIRE_PTR(hist_out, who);
    if (accept_len && (reinterpret_cast<uintptr_t>(accept_len) & 3u) != 0)
        return fail(GDN_ERR_INVALID_ARG, "%s: accept_len misaligned", who);
    const size_t el = shape->in_dtype == GDN_BF16 ? 2 : 4;
    const size_t qk = (size_t)shape->B * shape->T * shape->H_k * shape->d_k * el;
    const size_t vb = (size_t)shape->B * shape->T * shape->H_v * shape->d_v * el;
    const int64_t C = 2 * (int64_t)shape->H_k * shape->d_k + (int64_t)shape->H_v * shape->d_v;
    const size_t hb = (size_t)shape->B * (conv_k - 1) * C * el;
    if (hist_out && hist_out != hist_in && !overlap_ok(hist_out, hist_in, hb))
        return fail(GDN_ERR_INVALID_ARG, "%s: hist_out partially overlaps hist_in", who);
    if (outputs) {
        // every output region against every input region and the history
        const void* outs[3] = {q_out, k_out, v_out};
        const size_t osz[3] = {qk, qk, vb};
        const void* ins[5] = {q, k, v, hist_in, hist_out};
        const size_t isz[5] = {qk, qk, vb, hb, hb};
        for (int i = 0; i < 3; ++i)
            for (int j = 0; j < 5; ++j) {
                if (!ins[j]) continue;
                const char* a = static_cast<const char*>(outs[i]);
                const char* b = static_cast<const char*>(ins[j]);
                if (a < b + isz[j] && b < a + osz[i])
                    return fail(GDN_ERR_INVALID_ARG, "%s: an output overlaps an input or the history", who);
            }
    }
    gdn::ConvArgs c;
    memset(&c, 0, sizeof(c));
    c.q = q;
    c.k = k;
    c.v = v;
    c.w = conv_w;
    c.hist_in = hist_in;
    c.hist_out = hist_out;
    c.accept_len = accept_len;
    c.q_out = outputs ? q_out : nullptr;
    c.k_out = outputs ? k_out : nullptr;
    c.v_out = outputs ? v_out : nullptr;
    c.status_word = shape->status_word;
    c.B = shape->B;
    c.T = shape->T;
    c.C = (int)C;
    c.Cq = shape->H_k * shape->d_k;
    return launched(gdn::launch_short_conv(c, conv_k, shape->in_dtype == GDN_BF16, static_cast<cudaStream_t>(stream)),
                    who);
}

static gdn_status check_accept(const gdn_accept_shape* s, const char* who) {
    if (!s) return fail(GDN_ERR_INVALID_ARG, "%s: shape is NULL", who);
    if (s->B < 0 || s->T < 1 || s->V < 1)
        return fail(GDN_ERR_INVALID_ARG, "%s: sizes must be positive (B may be 0)", who);
    if (s->T > 16) return fail(GDN_ERR_UNSUPPORTED, "%s: T %d > 16", who, s->T);
    if (s->V % 8 != 0 || s->V > (1 << 18))
        return fail(GDN_ERR_UNSUPPORTED, "%s: V must be a multiple of 8 up to 2^18 (got %d)", who, s->V);
    if (s->B > (1 << 20)) return fail(GDN_ERR_UNSUPPORTED, "%s: B > 2^20", who);
    if (s->logits_dtype != GDN_F32 && s->logits_dtype != GDN_BF16)
        return fail(GDN_ERR_INVALID_ARG, "%s: logits_dtype %d unknown", who, s->logits_dtype);
    if (s->sampled != 0 && s->sampled != 1) return fail(GDN_ERR_INVALID_ARG, "%s: sampled must be 0 or 1", who);
    if (s->sampled && !(s->temperature > 0.f))
        return fail(GDN_ERR_INVALID_ARG, "%s: temperature must be > 0", who);
    return GDN_OK;
}

size_t gdn_accept_workspace_bytes(const gdn_accept_shape* shape) {
    if (check_accept(shape, "gdn_accept_workspace_bytes") != GDN_OK) return 0;
    return gdn::accept_workspace_bytes(shape->B, shape->T, shape->V, shape->sampled != 0);
}

gdn_status gdn_accept(const gdn_accept_shape* shape, const void* target_logits, const void* draft_logits,
                      const int32_t* tokens, const float* uniforms, int32_t* accept_len, int32_t* next_token,
                      void* workspace, size_t workspace_bytes, void* stream) {
    const char* who = "gdn_accept";
    gdn_status st = check_accept(shape, who);
    if (st != GDN_OK) return st;
    if (shape->B == 0) return ok();
    REQUIRE_PTR(target_logits, who);
    REQUIRE_PTR(tokens, who);
    REQUIRE_PTR(accept_len, who);
    REQUIRE_PTR(next_token, who);
    if (shape->sampled) {
        if (shape->T > 1) REQUIRE_PTR(draft_logits, who);
        REQUIRE_PTR(uniforms, who);
    }
    const size_t need = gdn::accept_workspace_bytes(shape->B, shape->T, shape->V, shape->sampled != 0);
    if (!workspace || workspace_bytes < need)
        return fail(GDN_ERR_WORKSPACE, "%s: workspace of %zu bytes needed", who, need);
    if (!aligned16(workspace)) return fail(GDN_ERR_INVALID_ARG, "%s: workspace not 16-byte aligned", who);
    gdn::AcceptArgs a = {};
    memset(&a, 0, sizeof(a));
    a.B = shape->B;
    a.T = shape->T;
    a.V = shape->V;
    a.bf16 = shape->logits_dtype == GDN_BF16;
    a.sampled = shape->sampled != 0;
    a.tau = shape->sampled ? shape->temperature : 1.f;
    a.target = target_logits;
    a.draft = draft_logits;
    a.tokens = tokens;
    a.u = uniforms;
    a.accept_len = accept_len;
    a.next_token = next_token;
    return launched(gdn::launch_accept(a, workspace, static_cast<cudaStream_t>(stream)), who);
}

gdn_status gdn_selftest_bounded_wait(int32_t* status_word, uint32_t polls, void* stream) {
    const char* who = "gdn_selftest_bounded_wait";
    if (!status_word || (reinterpret_cast<uintptr_t>(status_word) & 3u) != 0)
        return fail(GDN_ERR_INVALID_ARG, "%s: status_word is NULL or misaligned", who);
    if (polls == 0 || polls > (1u << 20)) return fail(GDN_ERR_INVALID_ARG, "%s: polls must be 1..2^20", who);
    return launched(gdn::launch_bounded_wait_selftest(status_word, polls, static_cast<cudaStream_t>(stream)), who);
}

gdn_status gdn_selftest_accept_wait(int32_t* status_word, int32_t* next_token, uint32_t polls, void* stream) {
    const char* who = "gdn_selftest_accept_wait";
    if (!status_word || (reinterpret_cast<uintptr_t>(status_word) & 3u) != 0)
        return fail(GDN_ERR_INVALID_ARG, "%s: status_word is NULL or misaligned", who);
    if (!next_token || (reinterpret_cast<uintptr_t>(next_token) & 3u) != 0)
        return fail(GDN_ERR_INVALID_ARG, "%s: next_token is NULL or misaligned", who);
    if (polls == 0 || polls > (1u << 20)) return fail(GDN_ERR_INVALID_ARG, "%s: polls must be 1..2^20", who);
    return launched(gdn::launch_accept_wait_selftest(status_word, next_token, polls, static_cast<cudaStream_t>(stream)),
                    who);
}

int32_t gdn_abi_version(void) { return GDN_ABI_VERSION; }

const char* gdn_last_verify_kernel(void) { return gdn::last_verify_kernel(); }

}  // extern "C"
