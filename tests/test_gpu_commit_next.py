"""GPU parity for gdn_commit_and_verify (commit-on-next-verify) against the fp64 oracle.

Two consecutive verify blocks on the same sequences: the first runs two-phase (stash only),
the second goes through gdn_commit_and_verify, which applies the first block's stash at its
accept counts and then runs the second block on the committed state. The oracle runs the two
blocks one after the other (each committed at its own counts). Both output forms are checked:
the second block committed at its counts in the same call, and the two-phase form (the state
ends at the committed first block, the second block's stash is committed later by
gdn_commit). Batches of 64 sequences take the single tensor-core kernel; batches of 2 take
the composed path (the commit kernel in place, then the verify kernel).
Tolerance: max |gpu - oracle| / max |oracle| <= 1e-4 per tensor."""
import numpy as np
import pytest
import torch

from gated_deltanet_mixer_verify_b200.inputs import make_inputs, workload
from gdn_helpers import TOL, oracle_verify, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn(cuda_device):
    from gated_deltanet_mixer_verify_b200 import build, gdn as g
    build.build()
    return g


def _stash(gdn, w):
    return torch.zeros(gdn.stash_bytes(w.B, w.T, w.H_k, w.H_v, w.d_k, w.d_v) // 4, dtype=torch.float32,
                       device="cuda")


def _case(gdn, B, seed, T2=8, two_phase_out=False, L1_set=None, gates="config"):
    w1 = workload("batched_verify", B=B, seed=seed)
    w2 = workload("batched_verify", B=B, seed=seed, T=T2)
    x1 = make_inputs(w1, layer=0, gates=gates)
    x2 = make_inputs(w2, layer=1, gates=gates)
    L1 = x1["accept_len"].numpy().copy()
    for i, v in (L1_set or {}).items():
        if i < B:
            L1[i] = v
    L2 = x2["accept_len"].numpy().copy()
    L2[0] = 0                                     # a rollback of the second block
    # Oracle: block 1 from S_base committed at L1 (out of range: rolled back), then block 2.
    L1_ok = np.where((L1 >= 0) & (L1 <= w1.T), L1, 0).astype(np.int32)
    _, S1_ref, _ = oracle_verify(x1, L1_ok)
    x2o = dict(x2)
    x2o["S0"] = torch.from_numpy(np.ascontiguousarray(S1_ref))
    o2_ref, S2_ref, _ = oracle_verify(x2o, L2)

    xd1, xd2 = to_dev(x1), to_dev(x2)
    state = xd1["S0"].clone()
    stash1 = _stash(gdn, w1)
    gdn.verify_step(xd1["q"], xd1["k"], xd1["v"], xd1["a"], xd1["b"], xd1["A_log"], xd1["dt_bias"],
                    state, None, None, stash=stash1)
    L1d = torch.as_tensor(L1).cuda()
    L2d = torch.as_tensor(L2).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if not two_phase_out:
        o2 = gdn.commit_and_verify(xd2["q"], xd2["k"], xd2["v"], xd2["a"], xd2["b"], xd2["A_log"],
                                   xd2["dt_bias"], state, stash1, L1d, w1.T, accept_len=L2d, status_word=status)
        torch.cuda.synchronize()
        assert rel_err(o2, o2_ref) <= TOL and rel_err(state, S2_ref) <= TOL
    else:
        stash2 = _stash(gdn, w2)
        o2 = gdn.commit_and_verify(xd2["q"], xd2["k"], xd2["v"], xd2["a"], xd2["b"], xd2["A_log"],
                                   xd2["dt_bias"], state, stash1, L1d, w1.T, accept_len=None, stash=stash2,
                                   status_word=status)
        torch.cuda.synchronize()
        assert rel_err(o2, o2_ref) <= TOL
        assert rel_err(state, S1_ref) <= TOL                  # the new base: block 1 committed
        gdn.commit(state, stash2, L2d, T=T2, H_k=w2.H_k)
        torch.cuda.synchronize()
        assert rel_err(state, S2_ref) <= TOL
    return int(status.item())


@pytest.mark.parametrize("B", [64, 2])
def test_commit_on_next_verify_fused(gdn, B):
    assert _case(gdn, B, seed=51, L1_set={1: 0, 2: 8}) == 0


@pytest.mark.parametrize("B", [64, 2])
def test_commit_on_next_verify_two_phase_again(gdn, B):
    assert _case(gdn, B, seed=52, two_phase_out=True, L1_set={0: 8, 3: 0}) == 0


def test_commit_on_next_verify_shorter_block_gentle_gates(gdn):
    # decays near 0.99: the first block's commit stays visible in the second block's outputs
    assert _case(gdn, 64, seed=53, T2=5, gates="gentle") == 0


def test_commit_on_next_verify_bad_previous_count_rolls_back(gdn):
    # an out-of-range previous count rolls that sequence back to its start and sets bit 1
    status = _case(gdn, 64, seed=54, L1_set={5: 9})
    assert status & 1
