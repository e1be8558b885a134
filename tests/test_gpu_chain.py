"""The verify -> accept -> commit chain on the GPU, with no accept count ever on the host: a
two-phase verify block writes its stash, gdn_accept turns the block's logits into device accept
counts, gdn_commit applies the stash at those counts and gdn_short_conv rewinds the filter
history at the same counts. Checked against the oracle run step by step (greedy acceptance is
exact, so the oracle's counts are the GPU's): committed state within the verify tolerance,
history bit-exact."""
import numpy as np
import pytest
import torch

from gated_deltanet_mixer_verify_b200.inputs import (as_f64, make_accept_inputs, make_conv_inputs,
                                                      make_inputs, workload)
from gdn_helpers import TOL, oracle_verify, rel_err, to_dev
from oracle import gdn_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn(cuda_device):
    from gated_deltanet_mixer_verify_b200 import build, gdn as g
    build.build()
    return g


@pytest.mark.parametrize("B", [64, 3])
def test_verify_accept_commit_on_device(gdn, B):
    w = workload("batched_verify", B=B, seed=91)
    x = make_inputs(w)
    acc = make_accept_inputs(w, V=4096)
    conv = make_conv_inputs(w)
    # oracle: the accept counts from the logits, then the block committed at them
    L_ref, nt_ref, _, _ = orc.accept(acc["target"].double().numpy(), acc["tokens"].numpy())
    _, S_ref, _ = oracle_verify(x, L_ref)
    f = as_f64(x)
    _, _, _, h_ref, _ = orc.short_conv(f["q"], f["k"], f["v"], conv["conv_w"].double().numpy(),
                                       conv["hist"].double().numpy(), L_ref)
    # GPU: verify two-phase, accept, commit and rewind at the device counts
    xd = to_dev(x)
    state = xd["S0"].clone()
    stash = torch.zeros(gdn.stash_bytes(w.B, w.T, w.H_k, w.H_v, w.d_k, w.d_v) // 4, device="cuda")
    gdn.verify_step(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"], state, None, None,
                    stash=stash)
    L_dev, nt_dev = gdn.accept(acc["target"].cuda(), acc["tokens"].cuda())
    gdn.commit(state, stash, L_dev, T=w.T, H_k=w.H_k)
    hist = conv["hist"].cuda()
    gdn.short_conv(xd["q"], xd["k"], xd["v"], None, hist, hist, L_dev, outputs=False)
    torch.cuda.synchronize()
    assert np.array_equal(L_dev.cpu().numpy(), L_ref) and np.array_equal(nt_dev.cpu().numpy(), nt_ref)
    assert rel_err(state, S_ref) <= TOL
    assert np.array_equal(hist.double().cpu().numpy(), h_ref)
    if B > 8:
        assert len(set(L_ref.tolist())) > 2
