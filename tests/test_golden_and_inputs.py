"""The stored oracle values reproduce, and the seeded generator is deterministic and
draws what it says (shapes, storage types, distributions, accept-length supports)."""
import json
import math
import os

import numpy as np
import pytest
import torch

from gated_deltanet_mixer_verify_b200.inputs import WORKLOADS, as_f64, make_inputs, workload
from oracle import gdn_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_verify_oracle.json")


def test_golden_tiny_verify_reproduces():
    g = json.load(open(GOLDEN))
    x = as_f64(make_inputs(workload("tiny_verify")))
    assert [int(v) for v in x["accept_len"]] == g["accept_len"]
    o, Sc, _ = orc.verify(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                          x["S0"], x["accept_len"])
    np.testing.assert_allclose(o.ravel(), g["o"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(Sc.ravel(), g["S_commit"], rtol=1e-13, atol=1e-15)


def test_generator_is_deterministic_and_layer_streams_differ():
    w = workload("batched_verify", B=2)
    x1, x2 = make_inputs(w, layer=3), make_inputs(w, layer=3)
    for key in x1:
        assert torch.equal(x1[key], x2[key])
    y = make_inputs(w, layer=4)
    assert not torch.equal(x1["q"], y["q"])


@pytest.mark.parametrize("name", ["tiny_verify", "batched_verify", "decode"])
def test_shapes_and_storage(name):
    w = workload(name, B=min(WORKLOADS[name].B, 4))
    x = make_inputs(w)
    dt = torch.float32 if w.in_dtype == "f32" else torch.bfloat16
    assert x["q"].shape == (w.B, w.T, w.H_k, w.d_k) and x["q"].dtype == dt
    assert x["k"].shape == (w.B, w.T, w.H_k, w.d_k) and x["k"].dtype == dt
    assert x["v"].shape == (w.B, w.T, w.H_v, w.d_v) and x["v"].dtype == dt
    assert x["a"].shape == (w.B, w.T, w.H_v) and x["b"].dtype == dt
    assert x["S0"].shape == (w.B, w.H_v, w.d_v, w.d_k) and x["S0"].dtype == torch.float32
    assert x["A_log"].shape == (w.H_v,) and x["dt_bias"].abs().max() == 0
    assert x["accept_len"].dtype == torch.int32 and x["accept_len"].shape == (w.B,)


def test_distributions():
    w = workload("batched_verify", B=16)
    x = make_inputs(w)
    s = x["S0"].double()
    assert abs(s.std().item() - 0.05) < 0.001 and abs(s.mean().item()) < 0.001
    q = x["q"].double()
    assert abs(q.std().item() - 1.0) < 0.02
    A = x["A_log"].double()
    assert A.min() >= 0.0 and A.max() <= math.log(16.0)
    big = make_inputs(workload("batched_verify", B=4096, H_k=1, H_v=1, d_k=1, d_v=1))["accept_len"].numpy()
    assert big.min() >= 1 and big.max() <= 8
    # P(L = 1) = 0.25 and P(L = 8) = 0.75^7 for the clipped geometric draw
    assert abs((big == 1).mean() - 0.25) < 0.03
    assert abs((big == 8).mean() - 0.75 ** 7) < 0.03
    tiny = np.array([int(make_inputs(workload("tiny_verify", seed=s))["accept_len"][0])
                     for s in range(400)])
    assert tiny.min() == 1 and tiny.max() == 8
    dec = make_inputs(workload("decode", B=8))
    assert dec["q"].shape[1] == 1 and (dec["accept_len"] == 1).all()
    pre = make_inputs(workload("prefill", T=128))
    assert pre["accept_len"] is None and pre["S0"].abs().max() == 0


def test_bf16_rounding_is_round_to_nearest_even():
    w = workload("batched_verify", B=1)
    x = make_inputs(w)
    # every stored value is a bf16 value: its float32 bit pattern has 16 zero low bits
    bits = x["q"].float().view(torch.int32)
    assert int((bits & 0xFFFF).abs().max()) == 0


def test_conv_inputs_shapes_ranges_and_streams():
    from gated_deltanet_mixer_verify_b200.inputs import make_conv_block, make_conv_inputs
    w = workload("batched_verify", B=3)
    C = 2 * w.H_k * w.d_k + w.H_v * w.d_v
    c = make_conv_inputs(w, K=4)
    assert c["conv_w"].shape == (C, 4) and c["conv_w"].dtype == torch.float32
    assert float(c["conv_w"].abs().max()) <= 0.5                     # U(-1/sqrt(K), 1/sqrt(K))
    assert c["hist"].shape == (3, 3, C) and c["hist"].dtype == torch.bfloat16
    blk = make_conv_block(w, K=3, layer=2)
    assert blk["q"].shape == (3, 8, 16, 128) and blk["v"].shape == (3, 8, 48, 128)
    assert blk["hist"].shape == (3, 2, C)
    assert 1 <= int(blk["accept_len"].min()) and int(blk["accept_len"].max()) <= 8
    # the mixer's own inputs are untouched by the convolution streams
    assert torch.equal(make_inputs(w)["q"], make_inputs(w)["q"])
    assert not torch.equal(make_conv_block(w, layer=2)["q"], make_conv_block(w, layer=3)["q"])
