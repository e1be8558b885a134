"""GPU parity for gdn_chunk_prefill against the fp64 per-token recurrence.

Tolerance: max |gpu - oracle| / max |oracle| <= 2e-3 per tensor (outputs; final state).
At the full 32768-token prompt the oracle recomputes a sample of value heads, each over
the whole prompt."""
import numpy as np
import pytest
import torch

from gated_deltanet_mixer_verify_b200.inputs import as_f64, make_inputs, workload
from gdn_helpers import TOL_BF16_OUT, TOL_PREFILL, rel_err, to_dev
from oracle import gdn_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn(cuda_device):
    from gated_deltanet_mixer_verify_b200 import build, gdn as g
    build.build()
    return g


def run_gpu(gdn, xd, state_in=None):
    o, S = gdn.chunk_prefill(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"],
                             xd["dt_bias"], state_in, None, None, 64)
    torch.cuda.synchronize()
    return o, S


@pytest.mark.parametrize("T,gates,with_state", [(300, "config", False), (300, "gentle", True),
                                                (64, "gentle", True), (1, "config", False),
                                                (1000, "gentle", False)])
def test_prefill_small_full_compare(gdn, T, gates, with_state):
    w = workload("prefill", T=T, H_k=2, H_v=6, seed=31 + T, state_std=0.05 if with_state else 0.0)
    x = make_inputs(w, gates=gates)
    f = as_f64(x)
    o_ref, S_ref = orc.prefill(f["q"], f["k"], f["v"], f["a"], f["b"], f["A_log"], f["dt_bias"],
                               f["S0"] if with_state else None)
    xd = to_dev(x)
    o, S = run_gpu(gdn, xd, xd["S0"] if with_state else None)
    assert rel_err(o, o_ref) <= TOL_PREFILL and rel_err(S, S_ref) <= TOL_PREFILL


def test_prefill_full_prompt_sampled_heads(gdn):
    w = workload("prefill")
    x = make_inputs(w)
    o, S = run_gpu(gdn, to_dev(x))
    G = w.H_v // w.H_k
    for h in (0, 25, 47):
        g = h // G
        sl = lambda t, lo, hi: t[:, :, lo:hi]
        f = as_f64({"q": sl(x["q"], g, g + 1), "k": sl(x["k"], g, g + 1),
                    "v": sl(x["v"], h, h + 1), "a": sl(x["a"], h, h + 1),
                    "b": sl(x["b"], h, h + 1), "A_log": x["A_log"][h:h + 1],
                    "dt_bias": x["dt_bias"][h:h + 1]})
        o_ref, S_ref = orc.prefill(f["q"], f["k"], f["v"], f["a"], f["b"], f["A_log"], f["dt_bias"])
        assert rel_err(o[:, :, h:h + 1], o_ref) <= TOL_PREFILL, h
        assert rel_err(S[:, h:h + 1], S_ref) <= TOL_PREFILL, h


def _oracle_prefill(x, with_state):
    f = as_f64(x)
    return orc.prefill(f["q"], f["k"], f["v"], f["a"], f["b"], f["A_log"], f["dt_bias"],
                       f["S0"] if with_state else None)


def test_prefill_long_gentle_decay_with_state(gdn):
    # Mild gates: the state's running decay crosses 2^-32 every dozen chunks or so, so the
    # kernel's lazy decay scalar and its occasional rescale of the stored state both run.
    w = workload("prefill", T=2048, H_k=1, H_v=2, seed=77, state_std=0.05)
    x = make_inputs(w, gates="gentle")
    o_ref, S_ref = _oracle_prefill(x, True)
    xd = to_dev(x)
    o, S = run_gpu(gdn, xd, xd["S0"])
    assert rel_err(o, o_ref) <= TOL_PREFILL and rel_err(S, S_ref) <= TOL_PREFILL


def test_prefill_fp32_inputs_bf16_outputs(gdn):
    w = workload("prefill", T=200, H_k=2, H_v=4, seed=78, in_dtype="f32", state_std=0.05)
    x = make_inputs(w, gates="gentle")
    o_ref, S_ref = _oracle_prefill(x, True)
    xd = to_dev(x)
    o, S = gdn.chunk_prefill(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"],
                             xd["S0"], None, None, 64, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert o.dtype == torch.bfloat16
    assert rel_err(o, o_ref) <= TOL_BF16_OUT and rel_err(S, S_ref) <= TOL_PREFILL


def test_prefill_batch_of_two_grouped_heads(gdn):
    # Two sequences, two value heads per key head: each key head's normalised tile is written
    # once and read by both of its value heads; a ragged last chunk (T % 64 = 3).
    w = workload("prefill", B=2, T=131, H_k=2, H_v=4, seed=79, state_std=0.05)
    x = make_inputs(w, gates="gentle")
    o_ref, S_ref = _oracle_prefill(x, True)
    xd = to_dev(x)
    o, S = run_gpu(gdn, xd, xd["S0"])
    assert rel_err(o, o_ref) <= TOL_PREFILL and rel_err(S, S_ref) <= TOL_PREFILL


def test_prefill_phases_match_the_one_call_prefill(gdn):
    # prepare then scan, each over the whole prompt, give the one-call prefill's bits (11
    # chunks: one piece); a second prompt prepared into its own workspace in between does not
    # disturb the first.
    w = workload("prefill", T=700, H_k=2, H_v=6, seed=80, state_std=0.05)
    x = to_dev(make_inputs(w, gates="gentle"))
    x2 = to_dev(make_inputs(workload("prefill", T=700, H_k=2, H_v=6, seed=81), gates="config"))
    o_ref, s_ref = run_gpu(gdn, x, x["S0"])
    nb = gdn.prefill_workspace_bytes(w.B, w.T, w.H_k, w.H_v, w.d_k, w.d_v)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    ws2 = torch.empty(nb, dtype=torch.uint8, device="cuda")
    gdn.chunk_prefill_prepare(x["q"], x["k"], x["a"], x["b"], x["A_log"], x["dt_bias"], ws)
    gdn.chunk_prefill_prepare(x2["q"], x2["k"], x2["a"], x2["b"], x2["A_log"], x2["dt_bias"], ws2)
    o, s = gdn.chunk_prefill_scan(x["v"], ws, w.H_k, x["S0"])
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(s, s_ref)


@pytest.mark.parametrize("T,pieces", [(4133, 2), (8197, 4)])
def test_prefill_in_pieces_matches_oracle(gdn, T, pieces):
    # 65 and 129 chunks, the last one ragged: the scan of each piece runs beside the preparation
    # of the next and starts from the state the previous piece left. Gentle gates and a nonzero
    # initial state, so the state carried across the piece boundaries is not decayed away.
    assert gdn.chunk_prefill_pieces(T) == pieces
    w = workload("prefill", T=T, H_k=1, H_v=3, seed=90 + pieces, state_std=0.05)
    x = make_inputs(w, gates="gentle")
    o_ref, S_ref = _oracle_prefill(x, True)
    xd = to_dev(x)
    o, S = run_gpu(gdn, xd, xd["S0"])
    assert rel_err(o, o_ref) <= TOL_PREFILL and rel_err(S, S_ref) <= TOL_PREFILL
    # in place (state_out = state_in): the same bits
    st = xd["S0"].clone()
    o2, _ = gdn.chunk_prefill(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"], st, st)
    torch.cuda.synchronize()
    assert torch.equal(o2, o) and torch.equal(st, S)


def test_prefill_in_pieces_is_ordered_on_the_callers_stream(gdn):
    # Work queued on the caller's stream after the call sees the finished outputs and state,
    # although the scans ran on the library's own stream.
    w = workload("prefill", T=8192, H_k=2, H_v=6, seed=95)
    xd = to_dev(make_inputs(w))
    o_ref, s_ref = run_gpu(gdn, xd)
    s = torch.cuda.Stream()
    o = torch.full(xd["v"].shape, float("nan"), device="cuda")
    st = torch.full((1, w.H_v, w.d_v, w.d_k), float("nan"), device="cuda")
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        gdn.chunk_prefill(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"], None, st, o)
        o_snap, s_snap = o.clone(), st.clone()
    torch.cuda.synchronize()
    assert torch.equal(o_snap, o_ref) and torch.equal(s_snap, s_ref)


def test_prefill_in_pieces_captures_into_a_cuda_graph(gdn):
    # Under capture the 4 pieces run in order on the capture stream (the library's shared side
    # stream never joins a capture), with the eager call's piece bounds: the replay gives the
    # eager call's bits.
    w = workload("prefill", T=8192, H_k=2, H_v=6, seed=96, state_std=0.05)
    xd = to_dev(make_inputs(w, gates="gentle"))
    o_ref, s_ref = run_gpu(gdn, xd, xd["S0"])          # eager (also creates the side stream)
    nb = gdn.prefill_workspace_bytes(w.B, w.T, w.H_k, w.H_v, w.d_k, w.d_v)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    o = torch.zeros_like(o_ref)
    st = torch.zeros_like(s_ref)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        gdn.chunk_prefill(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"], xd["S0"], st, o,
                          workspace=ws)                 # warm on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            gdn.chunk_prefill(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"], xd["S0"], st,
                              o, workspace=ws)
    o.zero_()
    st.zero_()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(st, s_ref)
    del g


def test_prefill_in_pieces_batch_of_two(gdn):
    # two sequences (the scan's grid carries the sequence index), 65 chunks each: 2 pieces,
    # the last chunk 4 tokens long
    w = workload("prefill", B=2, T=4100, H_k=1, H_v=2, seed=97, state_std=0.05)
    assert gdn.chunk_prefill_pieces(w.T) == 2
    x = make_inputs(w, gates="gentle")
    o_ref, S_ref = _oracle_prefill(x, True)
    xd = to_dev(x)
    o, S = run_gpu(gdn, xd, xd["S0"])
    assert rel_err(o, o_ref) <= TOL_PREFILL and rel_err(S, S_ref) <= TOL_PREFILL
