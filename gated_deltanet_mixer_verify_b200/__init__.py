"""Gated DeltaNet verify mixer for NVIDIA B200 (sm_100a).

The compute lives in ``libgdn.so`` (hand-written CUDA behind a C ABI, declared
in ``include/gdn.h``); :mod:`.gdn` is the thin ctypes binding over it and
:mod:`.inputs` the seeded synthetic-input generator. The binding is imported on
first use, so the input generator works on machines without the built library;
any call into the mixer raises if the library is missing.
"""

__all__ = ["verify_step", "commit", "decode_step", "chunk_prefill", "stash_bytes", "make_shape", "lib",
           "prefill_workspace_bytes", "GdnError", "library_path"]


def __getattr__(name):
    if name in __all__:
        from . import gdn
        return getattr(gdn, name)
    raise AttributeError(name)
