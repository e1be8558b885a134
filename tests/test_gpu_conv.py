"""GPU parity for gdn_short_conv (causal short convolution with its history rewound at device
accept counts) against the fp64 oracle, through the C ABI.

Tolerances, per element: fp32 outputs |gpu - oracle| <= 1e-5 max(1, |oracle|) (fp32 sums of
K products and one fp32 SiLU); bf16 outputs <= 2^-8 |oracle| + 1e-5 (one rounding to bf16,
half an 8-bit ulp, on top of the fp32 error). The history is a copy of inputs: bit-exact.
The chain convolution -> verify (fp32) meets the verify tolerance (1e-4 of the max)."""
import numpy as np
import pytest
import torch

from gated_deltanet_mixer_verify_b200.inputs import as_f64, make_conv_inputs, make_inputs, workload
from gdn_helpers import TOL, oracle_verify, rel_err, to_dev
from oracle import gdn_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn(cuda_device):
    from gated_deltanet_mixer_verify_b200 import build, gdn as g
    build.build()
    return g


def _check_out(gpu, ref, bf16):
    g = gpu.detach().double().cpu().numpy()
    r = np.asarray(ref, np.float64)
    bound = (2.0 ** -8) * np.abs(r) + 1e-5 if bf16 else 1e-5 * np.maximum(1.0, np.abs(r))
    bad = np.abs(g - r) > bound
    assert not bad.any(), "%d of %d elements out of bound, worst %g" % (bad.sum(), bad.size, np.max(np.abs(g - r) - bound))


def _run(gdn, w, K, L, inplace=True, seed_layer=0):
    x = make_inputs(w, layer=seed_layer)
    c = make_conv_inputs(w, K=K, layer=seed_layer)
    f = as_f64(x)
    qr, kr, vr, hr, bad = orc.short_conv(f["q"], f["k"], f["v"], c["conv_w"].double().numpy(),
                                         c["hist"].double().numpy(), L)
    xd = to_dev(x)
    w_d, h_d = c["conv_w"].cuda(), c["hist"].cuda()
    h_out = h_d if inplace else torch.full_like(h_d, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Ld = None if L is None else torch.as_tensor(np.asarray(L, np.int32)).cuda()
    q2, k2, v2 = gdn.short_conv(xd["q"], xd["k"], xd["v"], w_d, h_d, h_out, Ld, status_word=status)
    torch.cuda.synchronize()
    bf16 = w.in_dtype == "bf16"
    for gpu, ref in ((q2, qr), (k2, kr), (v2, vr)):
        _check_out(gpu, ref, bf16)
    assert np.array_equal(h_out.double().cpu().numpy(), hr)
    return int(status.item()), bad


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K", [2, 3, 4])
def test_verify_block_counts(gdn, dtype, K):
    # T = 8, accept counts 0 (rollback), 1, 2 (inside the old history), 5, 8 (all)
    w = workload("batched_verify", B=5, H_k=2, H_v=6, in_dtype=dtype, seed=71)
    status, bad = _run(gdn, w, K, np.array([0, 1, 2, 5, 8], np.int32))
    assert status == 0 and bad == 0


def test_full_size_batched_verify_shapes(gdn):
    # the benchmark's verify shapes: B = 64, H_k = 16, H_v = 48, d = 128, bf16, K = 4
    w = workload("batched_verify")
    L = make_inputs(w)["accept_len"].numpy()
    status, _ = _run(gdn, w, 4, L)
    assert status == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_shift(gdn, dtype):
    w = workload("decode", B=3, H_k=2, H_v=4, in_dtype=dtype, seed=72)
    assert _run(gdn, w, 4, None)[0] == 0                        # T = 1, no counts: shift by one


def test_short_block_keeps_part_of_history(gdn):
    # T = 2 < K - 1: the new history keeps old rows in front of the accepted inputs
    w = workload("batched_verify", B=3, T=2, H_k=1, H_v=2, in_dtype="f32", seed=73)
    assert _run(gdn, w, 4, np.array([0, 1, 2], np.int32), inplace=False)[0] == 0


@pytest.mark.parametrize("T", [33, 1000])
def test_long_prompt_tiles_and_rewind_launch(gdn, T):
    # several token tiles (ragged tail): the history is rewound by a second launch, in place
    w = workload("prefill", B=2, T=T, H_k=2, H_v=4, in_dtype="bf16", seed=74)
    assert _run(gdn, w, 4, None)[0] == 0


def test_out_of_range_count_keeps_history_and_sets_bit(gdn):
    w = workload("batched_verify", B=4, H_k=1, H_v=3, in_dtype="f32", seed=75)
    status, bad = _run(gdn, w, 4, np.array([9, -1, 3, 8], np.int32))
    assert bad == 2 and status & 1


def test_two_phase_history_rewind(gdn):
    # the convolution without a history write, then the rewind alone at the counts
    w = workload("batched_verify", B=4, H_k=2, H_v=6, in_dtype="bf16", seed=76)
    x, c = make_inputs(w), make_conv_inputs(w)
    f = as_f64(x)
    L = np.array([3, 0, 8, 1], np.int32)
    qr, kr, vr, hr, _ = orc.short_conv(f["q"], f["k"], f["v"], c["conv_w"].double().numpy(),
                                       c["hist"].double().numpy(), L)
    xd = to_dev(x)
    h_d = c["hist"].cuda()
    h_before = h_d.clone()
    q2, k2, v2 = gdn.short_conv(xd["q"], xd["k"], xd["v"], c["conv_w"].cuda(), h_d, None, None)
    torch.cuda.synchronize()
    assert torch.equal(h_d, h_before)                            # not written
    for gpu, ref in ((q2, qr), (k2, kr), (v2, vr)):
        _check_out(gpu, ref, True)
    gdn.short_conv(xd["q"], xd["k"], xd["v"], None, h_d, h_d, torch.as_tensor(L).cuda(), outputs=False)
    torch.cuda.synchronize()
    assert np.array_equal(h_d.double().cpu().numpy(), hr)


def test_conv_then_verify_chain(gdn):
    # fp32 end to end: the convolved q, k, v feed the verify mixer; state and history are both
    # committed at the same device counts.
    w = workload("batched_verify", B=8, H_k=4, H_v=12, in_dtype="f32", seed=77)
    x, c = make_inputs(w), make_conv_inputs(w)
    L = x["accept_len"].numpy().copy()
    L[0] = 0
    f = as_f64(x)
    qr, kr, vr, hr, _ = orc.short_conv(f["q"], f["k"], f["v"], c["conv_w"].double().numpy(),
                                       c["hist"].double().numpy(), L)
    o_ref, S_ref, _ = orc.verify(qr, kr, vr, f["a"], f["b"], f["A_log"], f["dt_bias"], f["S0"], L)
    xd = to_dev(x)
    h_d = c["hist"].cuda()
    Ld = torch.as_tensor(L).cuda()
    q2, k2, v2 = gdn.short_conv(xd["q"], xd["k"], xd["v"], c["conv_w"].cuda(), h_d, h_d, Ld)
    state = xd["S0"].clone()
    o = gdn.verify_step(q2, k2, v2, xd["a"], xd["b"], xd["A_log"], xd["dt_bias"], state, state, Ld)
    torch.cuda.synchronize()
    assert rel_err(o, o_ref) <= TOL and rel_err(state, S_ref) <= TOL
    assert np.array_equal(h_d.double().cpu().numpy(), hr)
