"""gdn_chunk_prefill_noalloc: the prefill for callers that cannot allocate device memory.

Some callers cannot pass the prefill a workspace, for example an engine whose memory
manager reserved all device memory at start-up, or a hot path that must stay out of the
CUDA allocator because cudaMalloc / cudaFree can synchronise the device. For them the
library keeps a fixed scratch array in its device code (64 MiB per GPU). These tests call
that entry point through the C ABI and check that its outputs match the ordinary,
workspace-taking gdn_chunk_prefill within the prefill tolerance, on two calls in a row that
share the scratch, and that a shape needing more scratch than there is gets a clear error.

This file is collected last on purpose: the scratch array is part of the library's device
code, so every test before it has already run when it is first used here."""
import ctypes

import numpy as np
import pytest
import torch

from gated_deltanet_mixer_verify_b200.inputs import make_inputs, workload
from gdn_helpers import TOL_PREFILL, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn(cuda_device):
    from gated_deltanet_mixer_verify_b200 import build, gdn as g
    build.build()
    return g


def _noalloc_call(gdn, x, state_in):
    """Call gdn_chunk_prefill_noalloc directly through the C ABI; the caller owns o and state."""
    lib = gdn.lib()
    B, T, H_k, d_k = x["k"].shape
    H_v, d_v = x["v"].shape[2], x["v"].shape[3]
    sh = gdn.make_shape(B, T, H_k, H_v, d_k, d_v, in_dtype=x["q"].dtype)
    o = torch.full(x["v"].shape, float("nan"), dtype=torch.float32, device="cuda")
    s_out = torch.full((B, H_v, d_v, d_k), float("nan"), dtype=torch.float32, device="cuda")
    p = lambda t: None if t is None else t.data_ptr()
    rc = lib.gdn_chunk_prefill_noalloc(ctypes.byref(sh), 64, p(x["q"]), p(x["k"]), p(x["v"]),
                                       p(x["a"]), p(x["b"]), p(x["A_log"]), p(x["dt_bias"]),
                                       p(state_in), p(s_out), p(o),
                                       torch.cuda.current_stream().cuda_stream)
    return rc, o, s_out


def test_noalloc_matches_workspace_prefill_on_two_calls(gdn):
    cases = [(workload("prefill", T=300, H_k=2, H_v=6, seed=41, state_std=0.0), "config", False),
             (workload("prefill", T=1000, H_k=1, H_v=3, seed=42, state_std=0.05), "gentle", True)]
    for w, gates, with_state in cases:
        x = to_dev(make_inputs(w, gates=gates))
        s_in = x["S0"] if with_state else None
        rc, o, s = _noalloc_call(gdn, x, s_in)
        assert rc == 0, gdn.lib().gdn_last_error().decode()
        o_ref, s_ref = gdn.chunk_prefill(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"],
                                         x["dt_bias"], s_in, None, None, 64)
        torch.cuda.synchronize()
        assert rel_err(o, o_ref.double().cpu().numpy()) <= TOL_PREFILL
        assert rel_err(s, s_ref.double().cpu().numpy()) <= TOL_PREFILL


def test_noalloc_rejects_shapes_beyond_its_scratch(gdn):
    # B = 1, H_v = 48 needs 49,728 bytes per 64-token chunk per head: 2048 tokens need 76 MiB.
    need = gdn.prefill_workspace_bytes(1, 2048, 16, 48, 128, 128)
    assert need > gdn.NOALLOC_SCRATCH_BYTES
    sh = gdn.make_shape(1, 2048, 16, 48, 128, 128)
    fake = 0x10000
    rc = gdn.lib().gdn_chunk_prefill_noalloc(ctypes.byref(sh), 64, *([fake] * 7), None, fake, fake,
                                            None)
    assert rc == -2
    msg = gdn.lib().gdn_last_error().decode()
    assert str(need) in msg and str(gdn.NOALLOC_SCRATCH_BYTES) in msg
