"""Gated DeltaNet verify mixer for NVIDIA B200 (sm_100a).

The compute lives in ``libgdn.so`` (hand-written CUDA behind a C ABI, declared
in ``include/gdn.h``); :mod:`.gdn` is the thin ctypes binding over it and
:mod:`.inputs` the seeded synthetic-input generator. The binding is imported on
first use, so the input generator works on machines without the built library;
any call into the mixer raises if the library is missing.
"""

__all__ = ["verify_step", "verify_step_gated", "commit", "commit_and_verify", "decode_step",
           "short_conv", "conv_channels", "gated_rmsnorm", "accept", "accept_workspace_bytes",
           "chunk_prefill", "chunk_prefill_prepare", "chunk_prefill_scan", "chunk_prefill_noalloc",
           "chunk_prefill_pieces", "prefill_workspace_bytes", "stash_bytes", "selftest_bounded_wait", "selftest_accept_wait",
           "make_shape", "lib", "last_verify_kernel", "GdnError", "library_path"]


def __getattr__(name):
    if name in __all__:
        from . import gdn
        return getattr(gdn, name)
    raise AttributeError(name)
