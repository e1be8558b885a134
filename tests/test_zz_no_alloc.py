"""gdn_chunk_prefill_noalloc: the prefill for callers that cannot allocate device memory.

Some callers cannot pass the prefill a workspace, for example an engine whose memory
manager reserved all device memory at start-up, or a hot path that must stay out of the
CUDA allocator because cudaMalloc / cudaFree can synchronise the device. For them the
library keeps a fixed scratch array in its device code (64 MiB per GPU). These tests call
that entry point through the C ABI and check, on two calls in a row that share the scratch,
that its outputs and final state match the fp64 oracle and the ordinary, workspace-taking
gdn_chunk_prefill within the prefill tolerance, on one-piece prompts and on one long enough
for the two-piece schedule (the scan on the library's side stream beside the next prepare).
They also check the exact size limit: the largest model-scale prompt that fits runs, one
chunk more gets a clear error.

The file is collected last so that a run that stops at its first failure has already run
every other test if one of these fails; the tests pass in any order, alone or after the
others."""
import ctypes

import pytest
import torch

from gated_deltanet_mixer_verify_b200.inputs import as_f64, make_inputs, workload
from gdn_helpers import TOL_PREFILL, rel_err, to_dev
from oracle import gdn_oracle as orc

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


def _oracle(x, with_state):
    f = as_f64(x)
    return orc.prefill(f["q"], f["k"], f["v"], f["a"], f["b"], f["A_log"], f["dt_bias"],
                       f["S0"] if with_state else None)


@pytest.mark.parametrize("T,H_k,H_v,gates,with_state", [
    (300, 2, 6, "config", False),      # 5 chunks, ragged last chunk
    (1000, 1, 3, "gentle", True),      # 16 chunks
    (4500, 1, 3, "gentle", True),      # 71 chunks: two pieces, ~15 MB of the scratch
])
def test_noalloc_matches_oracle_and_workspace_prefill_on_two_calls(gdn, T, H_k, H_v, gates, with_state):
    w = workload("prefill", T=T, H_k=H_k, H_v=H_v, seed=41 + T, state_std=0.05 if with_state else 0.0)
    x = make_inputs(w, gates=gates)
    o_ref, s_ref = _oracle(x, with_state)
    xd = to_dev(x)
    s_in = xd["S0"] if with_state else None
    if T >= 64 * 64:
        assert gdn.chunk_prefill_pieces(T, 64) == 2
    o_ws, s_ws = gdn.chunk_prefill(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"],
                                   xd["dt_bias"], s_in, None, None, 64)
    for call in range(2):                      # the second call reuses the scratch as left
        rc, o, s = _noalloc_call(gdn, xd, s_in)
        assert rc == 0, gdn.lib().gdn_last_error().decode()
        torch.cuda.synchronize()
        assert rel_err(o, o_ref) <= TOL_PREFILL and rel_err(s, s_ref) <= TOL_PREFILL, call
        assert rel_err(o, o_ws.double().cpu().numpy()) <= TOL_PREFILL, call
        assert rel_err(s, s_ws.double().cpu().numpy()) <= TOL_PREFILL, call


def test_noalloc_size_limit_at_model_scale(gdn):
    # Per 64-token chunk the scratch holds a 64 KB key/query tile per key head and a
    # 49,728-byte record per value head: 16 * 65,536 + 48 * 49,728 = 3,435,520 bytes at
    # H_k = 16, H_v = 48, so 19 chunks (1216 tokens) fit in 64 MiB and 20 chunks do not.
    per_chunk = 16 * 65536 + 48 * 49728
    assert gdn.prefill_workspace_bytes(1, 1216, 16, 48, 128, 128) == 19 * per_chunk
    assert 19 * per_chunk <= gdn.NOALLOC_SCRATCH_BYTES < 20 * per_chunk
    w = workload("prefill", T=1216, seed=45)
    x = make_inputs(w)
    xd = to_dev(x)
    rc, o, s = _noalloc_call(gdn, xd, None)
    assert rc == 0, gdn.lib().gdn_last_error().decode()
    o_ws, s_ws = gdn.chunk_prefill(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"],
                                   xd["dt_bias"], None, None, None, 64)
    torch.cuda.synchronize()
    assert rel_err(o, o_ws.double().cpu().numpy()) <= TOL_PREFILL
    assert rel_err(s, s_ws.double().cpu().numpy()) <= TOL_PREFILL
    # value head 47 (key head 15) against the oracle
    sl = lambda t, lo, hi: t[:, :, lo:hi]
    f = as_f64({"q": sl(x["q"], 15, 16), "k": sl(x["k"], 15, 16), "v": sl(x["v"], 47, 48),
                "a": sl(x["a"], 47, 48), "b": sl(x["b"], 47, 48), "A_log": x["A_log"][47:48],
                "dt_bias": x["dt_bias"][47:48]})
    o_ref, s_ref = orc.prefill(f["q"], f["k"], f["v"], f["a"], f["b"], f["A_log"], f["dt_bias"])
    assert rel_err(o[:, :, 47:48], o_ref) <= TOL_PREFILL and rel_err(s[:, 47:48], s_ref) <= TOL_PREFILL
    # one token more needs a 20th chunk: rejected on the host, before any launch
    need = gdn.prefill_workspace_bytes(1, 1217, 16, 48, 128, 128)
    assert need == 20 * per_chunk
    sh = gdn.make_shape(1, 1217, 16, 48, 128, 128)
    fake = 0x10000
    rc = gdn.lib().gdn_chunk_prefill_noalloc(ctypes.byref(sh), 64, *([fake] * 7), None, fake, fake,
                                            None)
    assert rc == -2
    msg = gdn.lib().gdn_last_error().decode()
    assert str(need) in msg and str(gdn.NOALLOC_SCRATCH_BYTES) in msg
