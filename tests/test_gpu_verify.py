"""GPU parity for gdn_verify_step / gdn_commit / gdn_decode_step against the fp64 oracle.

Every call goes through the C ABI (libgdn.so) via the ctypes binding; inputs are the
seeded synthetic workloads. Tolerance: max |gpu - oracle| / max |oracle| <= 1e-4 per
tensor (outputs; committed state); rollback is checked bit for bit."""
import json
import os

import numpy as np
import pytest
import torch

from gated_deltanet_mixer_verify_b200.inputs import make_inputs, workload
from gdn_helpers import (TOL, TOL_BF16_OUT, gpu_verify, launched_kernels, oracle_verify, rel_err, sm_count,
                         to_dev)

# The tensor-core kernels run when d_k = d_v = 128, 2 <= T <= 8 and there is at least one
# (sequence, value head) per SM: the persistent pipelined one (the kernel the batched-verify
# benchmark times) for a fused commit at device accept counts, the one-CTA-per-head one for the
# other forms (two-phase stash, commit-on-next-verify, gated norm).
PIPE_KERNEL = "gdn_verify_pipe_kernel"
TC_KERNEL = "gdn_verify_tc_kernel"


def on_tc_kernel(fn, B, H_v, kernel=PIPE_KERNEL):
    """Run fn (a verify call) and check that `kernel` is the one it launched."""
    assert B * H_v >= sm_count(), (B, H_v, sm_count())
    r, names = launched_kernels(fn)
    assert any(kernel in n for n in names), names
    return r

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn(cuda_device):
    from gated_deltanet_mixer_verify_b200 import build, gdn as g
    build.build()
    return g


def check(gdn, w, gates="config", accept=None, inplace=True, out_dtype=torch.float32, scale=1.0,
          tol=TOL):
    x = make_inputs(w, gates=gates, accept_len=accept)
    L = x["accept_len"].numpy()
    o_ref, S_ref, bad = oracle_verify(x, L, scale=scale)
    o, S = gpu_verify(gdn, to_dev(x), L, inplace=inplace, out_dtype=out_dtype, scale=scale)
    eo, es = rel_err(o, o_ref), rel_err(S, S_ref)
    assert eo <= tol and es <= TOL, (w.name, eo, es)
    return x, o, S


def test_tiny_verify_matches_oracle_and_golden(gdn):
    w = workload("tiny_verify")
    x, o, S = check(gdn, w)
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "tiny_verify_oracle.json")))
    assert rel_err(o.flatten(), np.array(g["o"])) <= TOL
    assert rel_err(S.flatten(), np.array(g["S_commit"])) <= TOL


def test_batched_verify_full_size(gdn):
    check(gdn, workload("batched_verify"))


def test_batched_verify_gentle_gates_out_of_place(gdn):
    # decays near 0.99: the initial state dominates the outputs and the commit
    check(gdn, workload("batched_verify", B=8), gates="gentle", inplace=False)


@pytest.mark.parametrize("layer", [0, 23, 47])
def test_single_sequence_model_scale_layers(gdn, layer):
    w = workload("single_seq_verify")
    L0 = make_inputs(w, layer=0)["accept_len"].numpy()        # one accept count per round
    x = make_inputs(w, layer=layer, accept_len=L0)
    o_ref, S_ref, _ = oracle_verify(x, L0)
    o, S = gpu_verify(gdn, to_dev(x), L0)
    assert rel_err(o, o_ref) <= TOL and rel_err(S, S_ref) <= TOL


def test_decode_full_size(gdn):
    w = workload("decode")
    x = make_inputs(w)
    o_ref, S_ref, _ = oracle_verify(x, None)
    xd = to_dev(x)
    state = xd["S0"].clone()
    o = gdn.decode_step(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"], state)
    torch.cuda.synchronize()
    assert rel_err(o, o_ref) <= TOL and rel_err(state, S_ref) <= TOL


@pytest.mark.parametrize("T", [1, 2, 3, 5, 7, 8, 9, 12, 16])
def test_every_block_length_and_accept_count(gdn, T):
    # 6 value heads per sequence: the small-batch latency kernel (T = 1 and 9..16 never reach
    # the tensor-core kernels at any size).
    w = workload("batched_verify", B=T + 1, T=T, H_k=2, H_v=6, seed=77 + T)
    accept = np.arange(T + 1, dtype=np.int32)                # every L in 0..T once
    check(gdn, w, gates="gentle", accept=accept)


@pytest.mark.parametrize("dk,dv,Hk,Hv", [(16, 16, 2, 2), (32, 32, 1, 3), (64, 64, 2, 4),
                                          (128, 40, 2, 6), (64, 100, 1, 1), (128, 1, 1, 2)])
def test_head_sizes_and_ragged_row_slices(gdn, dk, dv, Hk, Hv):
    w = workload("batched_verify", B=3, T=8, H_k=Hk, H_v=Hv, d_k=dk, d_v=dv, seed=dk + dv)
    check(gdn, w, gates="gentle", accept=np.array([8, 3, 1], np.int32), inplace=False)


def test_fp32_inputs_bf16_outputs_and_scale(gdn):
    w = workload("batched_verify", B=4, in_dtype="f32", seed=5)
    check(gdn, w, scale=128 ** -0.5)
    check(gdn, workload("batched_verify", B=4, seed=6), out_dtype=torch.bfloat16, tol=TOL_BF16_OUT)


@pytest.mark.parametrize("T", [2, 3, 4, 5, 6, 7, 8])
def test_tensor_core_kernel_every_block_length_and_accept_count(gdn, T):
    # Model-scale heads (H_k = 16, H_v = 48) and at least one head per SM, so that the
    # benchmarked tensor-core kernel runs; every L in 0..T, in place for even T.
    B = max(T + 1, 4)
    w = workload("batched_verify", B=B, T=T, seed=170 + T)
    accept = np.array([t % (T + 1) for t in range(B)], np.int32)
    x = make_inputs(w, gates="gentle", accept_len=accept)
    o_ref, S_ref, _ = oracle_verify(x, accept)
    xd = to_dev(x)
    o, S = on_tc_kernel(lambda: gpu_verify(gdn, xd, accept, inplace=T % 2 == 0), B, w.H_v)
    assert rel_err(o, o_ref) <= TOL and rel_err(S, S_ref) <= TOL
    assert torch.equal(S[0], xd["S0"][0])                    # L = 0: the state as it was


def test_rollback_is_bit_exact_in_and_out_of_place(gdn):
    B = 4
    w = workload("batched_verify", B=B, seed=9)
    x = make_inputs(w, accept_len=np.zeros(B, np.int32))
    xd = to_dev(x)
    for inplace in (True, False):
        _, S = on_tc_kernel(lambda: gpu_verify(gdn, xd, np.zeros(B, np.int32), inplace=inplace), B, w.H_v)
        assert torch.equal(S, xd["S0"])


def test_out_of_range_accept_commits_nothing_and_flags(gdn):
    B = 4
    w = workload("batched_verify", B=B, seed=10)
    x = make_inputs(w)
    xd = to_dev(x)
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    L = np.array([-1, 9, 4, 8], np.int32)
    o_ref, S_ref, bad = oracle_verify(x, L)
    assert list(bad) == [1, 1, 0, 0]
    for inplace in (True, False):
        status.zero_()
        o, S = on_tc_kernel(lambda: gpu_verify(gdn, xd, L, inplace=inplace, status=status), B, w.H_v)
        assert int(status[0].item()) & 1 == 1
        assert torch.equal(S[:2], xd["S0"][:2])
        assert rel_err(S[2:], S_ref[2:]) <= TOL and rel_err(o, o_ref) <= TOL
    status.zero_()
    gpu_verify(gdn, xd, np.array([8, 0, 4, 1], np.int32), status=status)
    assert int(status[0].item()) == 0


def test_out_of_range_accept_on_the_small_kernels(gdn):
    # 3 sequences x 48 heads is below one head per SM: the small-batch latency kernel runs.
    w = workload("batched_verify", B=3, seed=10)
    x = make_inputs(w)
    xd = to_dev(x)
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    L = np.array([-1, 9, 4], np.int32)
    o_ref, S_ref, bad = oracle_verify(x, L)
    for inplace in (True, False):
        status.zero_()
        o, S = gpu_verify(gdn, xd, L, inplace=inplace, status=status)
        assert int(status[0].item()) & 1 == 1
        assert torch.equal(S[:2], xd["S0"][:2])
        assert rel_err(S[2], S_ref[2]) <= TOL and rel_err(o, o_ref) <= TOL


def test_identity_gates_leave_state_bit_exact(gdn):
    # a = -1e4 gives alpha = 1 exactly and b = -1e4 gives beta = 0 exactly: S_L = S_0.
    B = 4
    L = np.array([8, 5, 1, 0], np.int32)
    w = workload("batched_verify", B=B, seed=11, in_dtype="f32")
    x = make_inputs(w, accept_len=L)
    x["a"].fill_(-1e4)
    x["b"].fill_(-1e4)
    xd = to_dev(x)
    _, S = on_tc_kernel(lambda: gpu_verify(gdn, xd, L, inplace=False), B, w.H_v)
    assert torch.equal(S.cpu(), x["S0"])


def test_write_then_read(gdn):
    # alpha = beta = 1 and q = k: o_t = S_t khat_t = v_t right after each write.
    B = 4
    w = workload("batched_verify", B=B, seed=12, in_dtype="f32")
    x = make_inputs(w)
    x["q"] = x["k"].clone()
    x["a"].fill_(-1e4)
    x["b"].fill_(1e4)
    xd = to_dev(x)
    o, _ = on_tc_kernel(lambda: gpu_verify(gdn, xd, x["accept_len"].numpy()), B, w.H_v)
    assert rel_err(o, x["v"].double().numpy()) <= 1e-5


def test_two_phase_commit_equals_fused(gdn):
    w = workload("batched_verify", B=16, seed=13)
    x = make_inputs(w)
    L = x["accept_len"].numpy().copy()
    L[:3] = [0, 8, 1]
    o_ref, S_ref, _ = oracle_verify(x, L)
    xd = to_dev(x)
    nbytes = gdn.stash_bytes(w.B, w.T, w.H_k, w.H_v, w.d_k, w.d_v)
    stash = torch.empty(nbytes // 4, dtype=torch.float32, device="cuda")
    state = xd["S0"].clone()
    o = on_tc_kernel(lambda: gdn.verify_step(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"],
                                             xd["dt_bias"], state, None, None, stash=stash),
                     w.B, w.H_v, kernel=TC_KERNEL)
    torch.cuda.synchronize()
    assert torch.equal(state, xd["S0"])                      # phase 1 leaves the state alone
    Ld = torch.as_tensor(L).cuda()
    out = torch.empty_like(state)
    gdn.commit(state, stash, Ld, T=w.T, H_k=w.H_k, state_out=out)
    gdn.commit(state, stash, Ld, T=w.T, H_k=w.H_k)            # in place
    torch.cuda.synchronize()
    assert rel_err(o, o_ref) <= TOL
    assert rel_err(out, S_ref) <= TOL and rel_err(state, S_ref) <= TOL
    assert torch.equal(state[0], xd["S0"][0])                # L = 0 in place: untouched
    _, S_fused = gpu_verify(gdn, xd, L)
    assert rel_err(S_fused, out.double().cpu().numpy()) <= TOL


def test_empty_batch(gdn):
    w = workload("batched_verify", B=1)
    x = to_dev(make_inputs(w))
    z = lambda t: t[:0]
    o = gdn.verify_step(z(x["q"]), z(x["k"]), z(x["v"]), z(x["a"]), z(x["b"]), x["A_log"],
                        x["dt_bias"], z(x["S0"]), None, z(x["accept_len"]))
    assert o.shape[0] == 0


@pytest.mark.parametrize("T", [1, 8, 16])
def test_latency_kernel_single_sequence(gdn, T):
    # One sequence of 48 heads (fewer heads than SMs): the latency kernel, checked against the
    # oracle for every accept count of the block in place, and a bad count and a rollback out
    # of place (bit for bit).
    w = workload("single_seq_verify", T=T, seed=200 + T)
    for L in range(T + 1):
        x = make_inputs(w, gates="gentle", accept_len=np.array([L], np.int32))
        o_ref, S_ref, _ = oracle_verify(x, x["accept_len"].numpy())
        xd = to_dev(x)
        (o, S), names = launched_kernels(lambda: gpu_verify(gdn, xd, np.array([L], np.int32), inplace=L > 0))
        assert any("gdn_verify_rec_kernel" in n for n in names), names
        if L == 0:
            assert torch.equal(S, xd["S0"])
        assert rel_err(o, o_ref) <= TOL and rel_err(S, S_ref) <= TOL, (T, L)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = make_inputs(w)
    xd = to_dev(x)
    o, S = gpu_verify(gdn, xd, np.array([T + 1], np.int32), inplace=False, status=status)
    assert int(status.item()) & 1 == 1 and torch.equal(S, xd["S0"])
