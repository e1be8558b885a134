"""Programmatic dependent launch (GDN_LAUNCH_PDL): the small-batch latency kernel (one sequence
of 48 heads) and the one-CTA-per-head kernel (decode of 4 sequences).

A layer loop launches one verify call per layer on one stream; with the flag each layer's
kernel may start while the previous layer's runs (it stages its own state first and waits for
that kernel before anything else). The results must be those of the plain launches, bit for
bit, eagerly and inside a CUDA graph, and match the fp64 oracle."""
import numpy as np
import pytest
import torch

from gated_deltanet_mixer_verify_b200.inputs import make_inputs, workload
from gdn_helpers import TOL, launched_kernels, oracle_verify, rel_err, to_dev

pytestmark = pytest.mark.gpu

LAYERS = 6


@pytest.fixture(scope="module")
def gdn(cuda_device):
    from gated_deltanet_mixer_verify_b200 import build, gdn as g
    build.build()
    return g


def _layers(w):
    L0 = make_inputs(w, layer=0)["accept_len"].numpy()       # one accept count per round
    xs = [make_inputs(w, layer=l, accept_len=L0, gates="gentle") for l in range(LAYERS)]
    return xs, [to_dev(x) for x in xs]


def _round(gdn, xds, pdl, states, outs):
    for xd, st, o in zip(xds, states, outs):
        gdn.verify_step(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"], st, st,
                        xd["accept_len"], o, pdl=pdl)


def test_pdl_layer_loop_matches_plain_launches_and_oracle(gdn):
    w = workload("single_seq_verify")
    xs, xds = _layers(w)
    res = {}
    for pdl in (False, True):
        states = [xd["S0"].clone() for xd in xds]
        outs = [torch.empty(xd["v"].shape, dtype=torch.float32, device="cuda") for xd in xds]
        _, names = launched_kernels(lambda: _round(gdn, xds, pdl, states, outs))
        assert any("gdn_verify_rec_kernel" in n for n in names), names
        res[pdl] = (states, outs)
    for l in range(LAYERS):
        assert torch.equal(res[True][0][l], res[False][0][l]), l
        assert torch.equal(res[True][1][l], res[False][1][l]), l
    L = xs[0]["accept_len"].numpy()
    o_ref, S_ref, _ = oracle_verify(xs[LAYERS - 1], L)
    assert rel_err(res[True][1][LAYERS - 1], o_ref) <= TOL and rel_err(res[True][0][LAYERS - 1], S_ref) <= TOL


def test_pdl_layer_loop_in_a_cuda_graph(gdn):
    w = workload("single_seq_verify")
    xs, xds = _layers(w)
    states = [xd["S0"].clone() for xd in xds]
    outs = [torch.empty(xd["v"].shape, dtype=torch.float32, device="cuda") for xd in xds]
    _round(gdn, xds, False, states, outs)                     # reference: two plain rounds
    _round(gdn, xds, False, states, outs)
    ref = ([s.clone() for s in states], [o.clone() for o in outs])
    s = torch.cuda.Stream()
    g_states = [xd["S0"].clone() for xd in xds]
    g_outs = [torch.empty_like(o) for o in outs]
    with torch.cuda.stream(s):
        _round(gdn, xds, True, g_states, g_outs)              # warm the launch path
    torch.cuda.synchronize()
    for st, xd in zip(g_states, xds):
        st.copy_(xd["S0"])
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        _round(gdn, xds, True, g_states, g_outs)
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    for l in range(LAYERS):
        assert torch.equal(g_states[l], ref[0][l]) and torch.equal(g_outs[l], ref[1][l]), l


def test_pdl_decode(gdn):
    w = workload("decode", B=4, seed=31)
    xd = to_dev(make_inputs(w))
    a, b = xd["S0"].clone(), xd["S0"].clone()
    o1 = gdn.decode_step(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"], a)
    o2, names = launched_kernels(lambda: gdn.decode_step(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"],
                                                         xd["dt_bias"], b, pdl=True))
    assert any("gdn_verify_head_kernel" in n for n in names), names
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(o1, o2)
