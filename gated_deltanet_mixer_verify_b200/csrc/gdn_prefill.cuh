// gdn_prefill.cuh -- long-prompt (chunked) prefill: shape rules, workspace size, launcher.
// Not part of the public interface.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "gdn.h"
#include "gdn_internal.cuh"

namespace gdn {

// 0 when this build supports the shape and chunk for prefill, -1 otherwise.
int check_prefill_shape(const gdn_shape* s, int chunk);

// Scratch bytes the prefill needs (0 when it needs none).
size_t prefill_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv, int chunk);

cudaError_t launch_prefill(const VerifyArgs& a, int chunk, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream);

// Pieces launch_prefill splits a T-token prompt into (0 for T <= 0); each is one preparation
// launch and one scan launch. Host-only.
int prefill_pieces(long long T);

// The two phases of the prefill, each over the whole prompt on one stream: the
// state-independent preparation (normalised keys / queries, per-chunk operators) into the
// workspace, then the sequential scan over the chunks, which reads it. (launch_prefill runs
// them piece by piece, the scan of one piece beside the preparation of the next.)
cudaError_t launch_prefill_prepare(const VerifyArgs& a, void* workspace, cudaStream_t stream);
cudaError_t launch_prefill_scan(const VerifyArgs& a, void* workspace, cudaStream_t stream);

// Size of the fixed device scratch behind gdn_chunk_prefill_noalloc (include/gdn.h).
constexpr size_t kNoAllocScratchBytes = GDN_NOALLOC_SCRATCH_BYTES;

// The prefill with its workspace in that fixed scratch; the caller checks the size.
cudaError_t launch_prefill_noalloc(const VerifyArgs& a, int chunk, cudaStream_t stream);

}  // namespace gdn
