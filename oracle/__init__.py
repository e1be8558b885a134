"""fp64 CPU oracle for the Gated DeltaNet verify mixer.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg import this package. The CUDA path
(``gated_deltanet_mixer_verify_b200``) never imports it, and it never imports
the CUDA path.
"""
