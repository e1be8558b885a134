/*
 * gdn.h -- C ABI of libgdn.so: the Gated DeltaNet layer mixer for speculative
 * verification, decode and long-prompt prefill on NVIDIA B200 (sm_100a).
 *
 * The operation (source pages: "Lithos-metal: Qwen3.8-27B on 40-core M5 Max",
 * table "GDN mixer" -- the recurrent state is split by value columns and each
 * slice is kept on-chip across the input block -- and its runtime paragraph,
 * where the GPU tracks recurrent-state commit and rollback; "Qwen 3.8 27B mac
 * m5: 200 tok/s, audited", section "How does lithos-metal fuse layer mixers on
 * Metal?" (a 32-bit recurrent state with a key side and a value side, which a
 * conventional kernel reads and writes for every token) and section "How does
 * DSpark speculative decoding create more than one token per read?" (7 drafted
 * tokens plus 1 anchor are verified as 8 rows; rewind follows acceptance)):
 *
 *   for each sequence b and value head h (key head g = h / (H_v / H_k)):
 *     khat_t = k_t / sqrt(|k_t|^2 + l2_eps),  qhat_t = scale * q_t / sqrt(|q_t|^2 + l2_eps)
 *     alpha_t = exp(-exp(A_log[h]) * softplus(a_t + dt_bias[h])),  beta_t = sigmoid(b_t)
 *     S_t = alpha_t S_{t-1} (I - beta_t khat_t khat_t^T) + beta_t v_t khat_t^T
 *     o_t = S_t qhat_t
 *   and the state committed for the block is S_L, L = accept_len[b] (L = 0: S_0).
 *
 * Layouts (all row-major, contiguous, no padding):
 *   q, k      [B][T][H_k][d_k]   in_dtype
 *   v         [B][T][H_v][d_v]   in_dtype
 *   a, b      [B][T][H_v]        in_dtype   (gate pre-activations)
 *   A_log     [H_v] fp32,  dt_bias [H_v] fp32
 *   state     [B][H_v][d_v][d_k] fp32       (row i = value index, column j = key index)
 *   o         [B][T][H_v][d_v]   out_dtype
 *   accept_len[B] int32, on the device
 *
 * Conventions shared by every call:
 *   - Every tensor pointer is a DEVICE pointer owned by the caller, and all
 *     tensor pointers must be 16-byte aligned. No call allocates or frees device
 *     memory; scratch comes from the caller (stash, workspace arguments). The
 *     library holds two pieces of state of its own, both for the life of the
 *     process:
 *       (1) a fixed device scratch array of GDN_NOALLOC_SCRATCH_BYTES (64 MiB),
 *           part of the library's device code, so that every GPU which loads the
 *           library holds it; only gdn_chunk_prefill_noalloc uses it;
 *       (2) per device, one non-blocking stream of the greatest priority and a
 *           few events, created on the first gdn_chunk_prefill (or _noalloc) of
 *           64 chunks or more on that device; the prompt's scans run there
 *           (see gdn_chunk_prefill).
 *     Every other call keeps nothing between calls.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *     is the legacy default stream). No call synchronises the host, and no call
 *     copies accept_len (or anything else) to the host.
 *   - Argument errors are detected on the host before anything is launched and
 *     returned as GDN_ERR_INVALID_ARG / GDN_ERR_UNSUPPORTED; nothing is written.
 *     GDN_ERR_CUDA means a launch failed (cudaGetLastError after the launch).
 *     gdn_last_error() gives a one-line reason for the last failure on the
 *     calling host thread.
 *   - Device-side conditions never trap: an accept_len[b] outside 0..T commits
 *     nothing for sequence b (its state_out equals state_in) and sets bit 0
 *     (GDN_STATUS_BAD_ACCEPT) of *status_word when status_word is not NULL.
 *   - Calls that overlap on the GPU and write the same buffers race; calls on
 *     one stream are ordered (gdn_chunk_prefill included, although a long
 *     prompt's scans run on a stream of the library's own: see there).
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* 10: gdn_selftest_accept_wait; 9: gdn_last_verify_kernel; 8: gdn_shape.launch_flags (GDN_LAUNCH_PDL); 7: prefill in pieces (gdn_chunk_prefill_pieces);
 * 6: gdn_accept; 5: gated norm; 4: gdn_short_conv; 3: commit-and-verify */
#define GDN_ABI_VERSION 10

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = -1,   /* bad shape, NULL or misaligned pointer, H_v % H_k != 0 */
    GDN_ERR_UNSUPPORTED = -2,   /* valid but not built: d_k / d_v / T / chunk outside the table */
    GDN_ERR_CUDA = -3,          /* a kernel launch failed */
    GDN_ERR_WORKSPACE = -4      /* workspace missing or smaller than the size query returns */
} gdn_status;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* Bits the kernels OR into *status_word. */
#define GDN_STATUS_BAD_ACCEPT 1     /* an accept_len[b] was outside 0..T: nothing committed for b */
#define GDN_STATUS_WAIT_TIMEOUT 2   /* a bounded wait for an asynchronous copy ran out: the
                                       affected heads were not written */

/*
 * Problem description shared by all calls. Sizes supported by this build:
 *   B in 0..65535, H_v a multiple of H_k, H_v <= 65535, B * H_v <= 2^24,
 *   d_k in {16, 32, 64, 128}, d_v in 1..4096,
 *   verify: T in 1..16; decode: T == 1; prefill: T >= 1, chunk == 64, d_k == d_v == 128.
 */
typedef struct {
    int32_t B, T, H_k, H_v, d_k, d_v;
    int32_t in_dtype;        /* gdn_dtype of q, k, v, a, b */
    int32_t out_dtype;       /* gdn_dtype of o */
    float l2_eps;            /* inside the square root of the q/k normalisation, e.g. 1e-6 */
    float scale;             /* multiplies qhat, e.g. 1.0 or 1/sqrt(d_k) */
    int32_t* status_word;    /* device int32 or NULL; bits GDN_STATUS_* are OR-ed in */
    uint32_t launch_flags;   /* 0, or GDN_LAUNCH_PDL (below) */
} gdn_shape;

/*
 * GDN_LAUNCH_PDL -- programmatic dependent launch for gdn_verify_step and gdn_decode_step on
 * the two small-batch kernels: the latency kernel (fewer (sequence, value head) pairs than
 * SMs, d_k = 128, T <= 16, fused commit) and the one-CTA-per-head kernel (the other small
 * batches, T = 1 and T > 8). The tensor-core kernels launch in plain stream order whatever
 * the flag says. The kernel may begin while the kernel launched just before it on the stream
 * is still running: it requests its state (state_in) and prefetches its q, k, v rows into L2
 * at once, and waits for that kernel to complete before it reads anything else or writes
 * anything. The caller guarantees that the kernel launched just before on the same stream
 * does not write state_in (in a layer loop each layer's state was last written by that
 * layer's previous call, long done; a loop of calls on one state must not set the flag).
 * It also lets the kernel after it start once its own inputs are staged. Works inside a
 * CUDA-graph capture.
 */
#define GDN_LAUNCH_PDL 1u

/*
 * gdn_verify_step -- one mixer pass over a verify block of T tokens (7 drafts +
 * 1 anchor is T = 8; the anchor is token 0), followed by the state commit.
 * Passages: the "GDN mixer" table and runtime paragraph of "Lithos-metal:
 * Qwen3.8-27B on 40-core M5 Max"; the DSpark section of "Qwen 3.8 27B mac m5:
 * 200 tok/s, audited" (8 verify rows, rewind after every acceptance decision).
 *
 *   o           out: o_t for all T tokens (outputs never depend on the commit point).
 *   accept_len  device [B] or NULL.
 *     non-NULL: fused commit. state_out[b] = S_L with L = accept_len[b]; L = 0 rolls
 *               back (state_out[b] = state_in[b] bit for bit; when state_out ==
 *               state_in nothing is written). state_out must not be NULL.
 *     NULL:     two-phase commit. The accept count is not known yet: stash receives
 *               what gdn_commit needs and state_out is not written (may be NULL).
 *   state_out   may equal state_in (in place); partial overlap is not allowed.
 *   stash       device, gdn_stash_bytes(shape) bytes; required when accept_len is NULL,
 *               optional (NULL or written) otherwise.
 */
gdn_status gdn_verify_step(const gdn_shape* shape,
                           const void* q, const void* k, const void* v,
                           const void* a, const void* b,
                           const float* A_log, const float* dt_bias,
                           const float* state_in, float* state_out,
                           const int32_t* accept_len,
                           void* o, float* stash, void* stream);

/*
 * gdn_commit -- second phase of a two-phase verify: once the accept count is known on
 * the device, state_out[b] = S_L built from the block's initial state and the stash
 * that gdn_verify_step wrote (accept_len NULL). Same passages as gdn_verify_step
 * (commit / rollback at the accepted prefix; rewind after acceptance).
 *   state_in   the state gdn_verify_step started from (unchanged since).
 *   state_out  may equal state_in. L = 0, or L out of range, leaves state_in's values.
 *   shape      the same shape that was passed to gdn_verify_step.
 */
gdn_status gdn_commit(const gdn_shape* shape, const float* state_in, float* state_out,
                      const float* stash, const int32_t* accept_len, void* stream);

/*
 * gdn_decode_step -- plain decoding, one token (shape->T must be 1): o = S_1 q and the
 * state is updated in place (always committed). This is the case the pages describe as
 * a conventional kernel reading and writing the whole state for every token ("Qwen 3.8
 * 27B mac m5: 200 tok/s, audited", section on fusing layer mixers).
 */
gdn_status gdn_decode_step(const gdn_shape* shape,
                           const void* q, const void* k, const void* v,
                           const void* a, const void* b,
                           const float* A_log, const float* dt_bias,
                           float* state, void* o, void* stream);

/*
 * gdn_commit_and_verify -- commit-on-next-verify: the previous block's two-phase commit is
 * folded into the next verify block, so that the state is read once and written once per
 * block even when the accept count is not known at verify time. Passages: the GPU-resident
 * commit / rollback ("Lithos-metal: Qwen3.8-27B on 40-core M5 Max", runtime paragraph) and
 * the rewind after every acceptance decision ("Qwen 3.8 27B mac m5: 200 tok/s, audited",
 * section "How does DSpark speculative decoding create more than one token per read?").
 *   shape            this block's shape (T tokens).
 *   prev_T           the previous block's T (1..16): the layout of prev_stash.
 *   state            in: the state the previous block started from (what that block's
 *                    gdn_verify_step read); out: see accept_len. [B][H_v][d_v][d_k] fp32.
 *   prev_stash       what that gdn_verify_step wrote as its stash (two-phase, accept_len NULL).
 *   prev_accept_len  [B] int32, device: that block's accept counts (0..prev_T; out of range
 *                    rolls the sequence back to its start and sets status bit 1).
 *   accept_len       this block's accept counts (device) or NULL:
 *                    given: state <- this block committed at accept_len (both commits applied);
 *                    NULL:  state <- the previous block committed at prev_accept_len (the new
 *                           base), and stash <- this block's stash, for the next call.
 *   o, stash         as gdn_verify_step; this block's outputs see the committed previous state.
 * With d_k = d_v = 128, 2 <= T <= 8, prev_T <= 8 and B * H_v at least the SM count, one kernel
 * does all of it; other shapes run gdn_commit's kernel in place first (one more state pass).
 */
gdn_status gdn_commit_and_verify(const gdn_shape* shape, int32_t prev_T,
                                 const void* q, const void* k, const void* v,
                                 const void* a, const void* b,
                                 const float* A_log, const float* dt_bias,
                                 float* state, const float* prev_stash, const int32_t* prev_accept_len,
                                 const int32_t* accept_len, void* o, float* stash, void* stream);

/*
 * gdn_chunk_prefill -- the mixer over a long prompt (T tokens per sequence), in the
 * chunked WY / UT-transform form on tensor cores: o for every token and the state after
 * the last token. The pages time whole-model prefill only ("Qwen 3.8 27B mac m5: 200
 * tok/s, audited", section "What does long-context prefill cost on Apple silicon?");
 * the recurrence is the one above.
 *   state_in   NULL = zero initial state.
 *   state_out  required; may equal state_in.
 *   workspace  device scratch of at least gdn_chunk_prefill_workspace_bytes(shape, chunk)
 *              bytes (16-byte aligned); contents on entry are ignored.
 * Streams: a prompt of 64 chunks or more is split into gdn_chunk_prefill_pieces(T, chunk)
 * pieces of whole chunks. The scan of piece i runs on a stream of the greatest priority that
 * the library creates per device on first use (non-blocking), beside the preparation of piece
 * i + 1 on `stream`; events order the pieces and join that stream back to `stream` before the
 * call returns, so work queued on `stream` afterwards sees the finished o and state_out. The
 * first such call on a device creates the stream and its events. Calls from several host
 * threads are serialised while they queue their launches, and their scans share that stream.
 * While `stream` is being captured into a CUDA graph, the pieces run in order on `stream`
 * alone (same piece bounds, same results; the shared stream never joins a capture, so an
 * eager call from another thread cannot land in the graph).
 */
gdn_status gdn_chunk_prefill(const gdn_shape* shape, int32_t chunk,
                             const void* q, const void* k, const void* v,
                             const void* a, const void* b,
                             const float* A_log, const float* dt_bias,
                             const float* state_in, float* state_out, void* o,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * gdn_chunk_prefill_prepare / gdn_chunk_prefill_scan -- the two phases of gdn_chunk_prefill,
 * each over the whole prompt on the given stream, for callers that schedule them separately (for instance the
 * preparation of the next prompt alongside the scan of this one, or timing each phase). Same
 * recurrence and chunk algebra as gdn_chunk_prefill; the split itself has no counterpart in
 * the source pages.
 *   prepare  reads q, k [B,T,H_k,d_k], a, b [B,T,H_v], A_log, dt_bias [H_v] and writes every
 *            per-chunk operator the scan needs into the workspace: the normalised keys and
 *            queries once per (sequence, key head, chunk), and per (sequence, value head,
 *            chunk) the decays, the write strengths and the chunk's output / state-update
 *            operators. No state is read. Chunks are independent and run in parallel.
 *   scan     reads v [B,T,H_v,d_v], state_in (NULL = zero), the prepared workspace, and writes
 *            o and state_out exactly as gdn_chunk_prefill does; it walks the chunks in order.
 * The shape (including H_k, which lays out the workspace), chunk, workspace and
 * workspace_bytes must be the same in both calls, and the scan must be ordered after the
 * prepare (same stream, or an event between them). The workspace belongs to the caller and
 * must not be reused by another call until the scan has completed. Errors are those of
 * gdn_chunk_prefill (GDN_ERR_WORKSPACE for a missing or short workspace).
 */
gdn_status gdn_chunk_prefill_prepare(const gdn_shape* shape, int32_t chunk,
                                     const void* q, const void* k,
                                     const void* a, const void* b,
                                     const float* A_log, const float* dt_bias,
                                     void* workspace, size_t workspace_bytes, void* stream);
gdn_status gdn_chunk_prefill_scan(const gdn_shape* shape, int32_t chunk,
                                  const void* v, const float* state_in, float* state_out, void* o,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* Size of the fixed device scratch behind gdn_chunk_prefill_noalloc: 64 MiB. */
#define GDN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * gdn_chunk_prefill_noalloc -- gdn_chunk_prefill for callers that cannot allocate device
 * memory. (The source pages have no counterpart; this is a convenience of this library.)
 *
 * Some callers cannot hand the prefill a workspace: an engine whose memory manager reserved
 * all device memory at start-up and will not give out more, or a hot path that must not
 * enter the CUDA allocator because cudaMalloc / cudaFree can synchronise the device and stall
 * every stream. This entry point takes the same arguments as gdn_chunk_prefill minus the
 * workspace, and uses a fixed scratch array that is part of the library's device code instead:
 *   - The scratch is GDN_NOALLOC_SCRATCH_BYTES. Every GPU that loads the library keeps it
 *     allocated until the process exits, whether or not this entry point is called.
 *   - Shapes whose workspace (gdn_chunk_prefill_workspace_bytes) exceeds it are rejected with
 *     GDN_ERR_UNSUPPORTED and a gdn_last_error() message giving both sizes; with d = 128 and
 *     chunk 64 each 64-token chunk of a sequence needs 49,728 bytes per value head plus
 *     65,536 bytes per key head, e.g. up to 19 chunks (1,216 tokens) for B = 1, H_v = 48 and
 *     H_k = 16.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - All calls on one GPU share the same scratch and it keeps the last call's contents.
 *     Nothing in it needs to start at zero (each call writes every element it later reads),
 *     but calls that may overlap on the GPU -- on different streams without ordering between
 *     them -- race on the scratch and can corrupt each other's results. Order them.
 *   - The first call on a device looks up the scratch's device address (once per device,
 *     with that device current); make that first call before any stream capture.
 */
gdn_status gdn_chunk_prefill_noalloc(const gdn_shape* shape, int32_t chunk,
                                     const void* q, const void* k, const void* v,
                                     const void* a, const void* b,
                                     const float* A_log, const float* dt_bias,
                                     const float* state_in, float* state_out, void* o,
                                     void* stream);

/*
 * gdn_verify_step_gated -- gdn_verify_step with the mixer's output gating and normalisation
 * ("Lithos-metal: Qwen3.8-27B on 40-core M5 Max", table "GDN mixer": projections, recurrence,
 * gating and normalisation in one mixer; the formula is the plain reading of it): every output
 * row (one token of one value head, d_v values) becomes
 *   o <- o / sqrt(mean(o^2) + norm_eps) * norm_w * silu(norm_z)
 *   norm_z     [B][T][H_v][d_v] in_dtype (the layout of v): the gate input. Required.
 *   norm_w     [d_v] fp32, shared by all heads.
 *   norm_eps   >= 0 (e.g. 1e-6), inside the square root.
 * Statistics are fp32. The tensor-core verify kernel applies it to its outputs in registers
 * (one extra read of norm_z); other shapes run the mixer, then gdn_gated_rmsnorm over o in
 * place (from o as stored in out_dtype). d_v must be a multiple of 4. Everything else is as
 * gdn_verify_step, whose stash and state are unaffected.
 */
gdn_status gdn_verify_step_gated(const gdn_shape* shape,
                                 const void* q, const void* k, const void* v,
                                 const void* a, const void* b,
                                 const float* A_log, const float* dt_bias,
                                 const float* state_in, float* state_out,
                                 const int32_t* accept_len,
                                 const void* norm_z, const float* norm_w, float norm_eps,
                                 void* o, float* stash, void* stream);

/*
 * gdn_gated_rmsnorm -- the same gated RMS normalisation as a standalone pass over any mixer
 * output (decode, prefill): rows of d elements,
 *   y = x / sqrt(mean(x^2) + eps) * w * silu(z)
 *   x, z, y    [rows][d] with dtypes x_dtype, z_dtype, y_dtype (GDN_F32 or GDN_BF16);
 *              y may be x (in place, same dtype) but must not partially overlap it.
 *   w          [d] fp32.   d: a multiple of 4, up to 4096.   eps >= 0.
 * One warp per row, statistics in fp32.
 */
gdn_status gdn_gated_rmsnorm(int64_t rows, int32_t d, const void* x, int32_t x_dtype,
                             const void* z, int32_t z_dtype, const float* w, float eps,
                             void* y, int32_t y_dtype, void* stream);

/*
 * gdn_short_conv -- the causal short convolution in front of the mixer (one filter of conv_k
 * taps per channel, SiLU after the sum, no bias) with the filter's short history, rewound to
 * the accepted prefix. That history is one of the three structures brought back in line with
 * the accepted tokens after a verify block ("Qwen 3.8 27B mac m5: 200 tok/s, audited",
 * section "How does DSpark speculative decoding create more than one token per read?"); the
 * page fixes no width or activation, and this is the plain reading of it.
 * Channels are ordered q | k | v: C = 2 H_k d_k + H_v d_v; channel g d_k + j is q head g,
 * column j; H_k d_k + g d_k + j is k; 2 H_k d_k + h d_v + j is v. Per sequence b, channel c:
 *   xc = [hist_in rows 0 .. conv_k - 2 (oldest first), the block's inputs x_0 .. x_{T-1}]
 *   out_t = silu(sum_{i < conv_k} conv_w[c][i] xc[t + i])   (conv_w[c][conv_k - 1] weighs x_t)
 *   hist_out rows = xc[L .. L + conv_k - 2],  L = accept_len[b] (L = T when accept_len is NULL)
 *   shape          B, T, H_k, H_v, d_k, d_v, in_dtype (inputs, outputs and history alike) and
 *                  status_word; d_k and d_v multiples of 8; T up to 2^20.
 *   conv_k         filter taps: 2, 3 or 4 (else GDN_ERR_UNSUPPORTED).
 *   q, k, v        the block's inputs before the convolution, layouts as gdn_verify_step.
 *   conv_w         [C][conv_k] fp32.
 *   hist_in        [B][conv_k - 1][C] in_dtype: the last conv_k - 1 inputs before the block.
 *   hist_out       same layout, or NULL (history not written: two-phase, rewind later by a
 *                  call with NULL outputs). May equal hist_in (rewound in place).
 *   accept_len     [B] int32, device, or NULL. An out-of-range count keeps the old history
 *                  and sets status bit 1 (GDN_STATUS_BAD_ACCEPT).
 *   q_out, k_out, v_out  the convolved q, k, v (layouts of q, k, v), all given or all NULL
 *                  (history rewind only). They must not overlap the inputs or the history.
 * Everything is caller-owned device memory, 16-byte aligned. The arithmetic is fp32; outputs
 * are rounded once to in_dtype. History rows are copies of inputs, so a rewind is exact.
 * Returns GDN_ERR_INVALID_ARG when q_out, k_out, v_out and hist_out are all NULL.
 */
gdn_status gdn_short_conv(const gdn_shape* shape, int32_t conv_k,
                          const void* q, const void* k, const void* v, const float* conv_w,
                          const void* hist_in, void* hist_out, const int32_t* accept_len,
                          void* q_out, void* k_out, void* v_out, void* stream);

/*
 * gdn_accept -- device-side acceptance of verify blocks, so that verify -> accept -> commit
 * never leaves the GPU ("Lithos-metal: Qwen3.8-27B on 40-core M5 Max", runtime paragraph on
 * GPU-resident commit / rollback; "Qwen 3.8 27B mac m5: 200 tok/s, audited", section "How does
 * DSpark speculative decoding create more than one token per read?": exact speculative
 * sampling, greedy or sampled, then a correction or a bonus token).
 *   tokens          [B][T] int32: row 0 the anchor (the last confirmed token), rows 1..T-1 drafts.
 *   target_logits   [B][T][V] logits_dtype: row t is the large model's prediction of the token
 *                   after row t.
 *   draft_logits    [B][T-1][V] logits_dtype (sampled mode; NULL for greedy): row t is the
 *                   drafter's prediction that proposed draft t+1.
 *   uniforms        [B][T] fp32 in [0, 1) (sampled mode; NULL for greedy): uniforms[b][t+1]
 *                   decides draft t+1, uniforms[b][0] draws the next token.
 *   accept_len      [B] int32 out: 1 + the number of leading drafts that survive (1..T): the
 *                   block rows the mixer commits (its accept_len argument, on the device).
 *   next_token      [B] int32 out: greedy, the argmax at row n (the first rejected row, or the
 *                   last row); sampled, a draw with uniforms[b][0] from max(0, p_n - q_n)
 *                   normalised (a rejection) or from p_{T-1} (every draft survived).
 * p_t = softmax(target_t / temperature), q_t = softmax(draft_t / temperature). Greedy keeps
 * draft t+1 iff it is the first index of the maximum of target row t; sampled keeps it iff
 * uniforms[b][t+1] * q_t(d) < p_t(d). Decisions are taken in fp32. A draw takes the first index
 * whose running mass exceeds u times the total. workspace: gdn_accept_workspace_bytes, 16-byte
 * aligned, contents irrelevant (the call zeroes what it needs). V a multiple of 8, up to 2^18;
 * T 1..16.
 */
typedef struct {
    int32_t B, T, V;
    int32_t logits_dtype;    /* GDN_F32 or GDN_BF16, for both logit arrays */
    int32_t sampled;         /* 0: greedy; 1: exact speculative sampling */
    float temperature;       /* > 0 (sampled mode) */
} gdn_accept_shape;

gdn_status gdn_accept(const gdn_accept_shape* shape, const void* target_logits, const void* draft_logits,
                      const int32_t* tokens, const float* uniforms, int32_t* accept_len, int32_t* next_token,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace gdn_accept needs (0 for an invalid shape). */
size_t gdn_accept_workspace_bytes(const gdn_accept_shape* shape);

/* Bytes of stash gdn_verify_step writes for this shape (0 for an invalid shape). */
size_t gdn_stash_bytes(const gdn_shape* shape);

/* Bytes of workspace gdn_chunk_prefill (and each of its two phases) needs (0 for an invalid
 * shape or chunk): per sequence and 64-token chunk, 65,536 bytes per key head and 49,728 per
 * value head. */
size_t gdn_chunk_prefill_workspace_bytes(const gdn_shape* shape, int32_t chunk);

/* Pieces gdn_chunk_prefill splits a T-token prompt into, each one preparation launch and one
 * scan launch: with n = ceil(T / chunk) chunks, min(4, max(1, n / 32)) (integer division), so
 * 1 below 64 chunks and 4 from 128; 0 for T = 0; -1 for T < 0 or an unsupported chunk. */
int32_t gdn_chunk_prefill_pieces(int64_t T, int32_t chunk);

/*
 * gdn_selftest_bounded_wait -- test hook for the failure path that every bounded mbarrier wait
 * in the library shares: one kernel waits, with the same helper, on an mbarrier that nothing
 * completes;
 * after `polls` polls (1..2^20) it gives up, ORs GDN_STATUS_WAIT_TIMEOUT into *status_word
 * (device int32) and returns. The context stays usable. Nothing faults, traps or hangs.
 */
gdn_status gdn_selftest_bounded_wait(int32_t* status_word, uint32_t polls, void* stream);

/*
 * gdn_selftest_accept_wait -- test hook for the other kind of bounded wait: gdn_accept's draw
 * kernel waits for its sequence's flag, raised by the row kernel's last row of the sequence.
 * Here the draw kernel runs alone for one sequence whose flag nothing raises; each of its CTAs
 * gives up after `polls` polls (1..2^20), ORs GDN_STATUS_WAIT_TIMEOUT into *status_word and
 * writes 0 to next_token[0] (both device int32), and touches nothing else. The context stays
 * usable. Nothing faults, traps or hangs.
 */
gdn_status gdn_selftest_accept_wait(int32_t* status_word, int32_t* next_token, uint32_t polls, void* stream);

/* Static description of a status code. */
const char* gdn_status_string(gdn_status status);

/* One-line reason for the most recent failing call on this host thread ("" if none). */
const char* gdn_last_error(void);

/* GDN_ABI_VERSION of the built library. */
int32_t gdn_abi_version(void);

/*
 * Name of the mixer kernel that the calling host thread's most recent gdn_verify_step,
 * gdn_verify_step_gated, gdn_decode_step or gdn_commit_and_verify chose to launch (for
 * example "gdn_verify_pipe_kernel"; "" before the first such call). The name is that of the
 * CUDA kernel function. The string is static; the caller does not free it.
 */
const char* gdn_last_verify_kernel(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
