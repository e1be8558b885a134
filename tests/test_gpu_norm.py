"""GPU parity for the gated RMS normalisation of the mixer output against the fp64 oracle,
through the C ABI: the standalone pass (gdn_gated_rmsnorm) element by element, and the verify
mixer with the normalisation applied (gdn_verify_step_gated) on the tensor-core kernel (fused,
B*H_v >= the SM count) and on the composed path (mixer, then the standalone pass).

Tolerances: standalone, per element, fp32 output |gpu - oracle| <= 1e-5 max(1, |oracle|)
(fp32 statistics, rsqrt and exp approximations at ~1e-6); bf16 output 2^-8 |oracle| + 1e-5
(one rounding). The verify mixer with the normalisation: max |gpu - oracle| / max |oracle|
<= 1e-4 per tensor for fp32 outputs (the verify tolerance), 8e-3 for bf16 outputs; the
committed state as for verify."""
import numpy as np
import pytest
import torch

from gated_deltanet_mixer_verify_b200.inputs import as_f64, make_inputs, make_norm_inputs, workload
from gdn_helpers import TOL, TOL_BF16_OUT, oracle_verify, rel_err, to_dev
from oracle import gdn_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn(cuda_device):
    from gated_deltanet_mixer_verify_b200 import build, gdn as g
    build.build()
    return g


def _check(gpu, ref, bf16):
    g = gpu.detach().double().cpu().numpy()
    r = np.asarray(ref, np.float64)
    bound = (2.0 ** -8) * np.abs(r) + 1e-5 if bf16 else 1e-5 * np.maximum(1.0, np.abs(r))
    bad = np.abs(g - r) > bound
    assert not bad.any(), "%d of %d out of bound, worst excess %g" % (bad.sum(), bad.size, np.max(np.abs(g - r) - bound))


@pytest.mark.parametrize("d", [128, 64, 1000, 2048])
@pytest.mark.parametrize("xt,zt,yt", [(torch.float32, torch.bfloat16, torch.float32),
                                      (torch.float32, torch.bfloat16, torch.bfloat16),
                                      (torch.bfloat16, torch.float32, torch.float32)])
def test_standalone_matches_oracle(gdn, d, xt, zt, yt):
    r = np.random.default_rng(d)
    rows = 37
    x = torch.from_numpy(r.standard_normal((rows, d)).astype(np.float32) * 0.3).to(xt)
    z = torch.from_numpy(r.standard_normal((rows, d)).astype(np.float32)).to(zt)
    w = torch.from_numpy(r.uniform(0.5, 1.5, d).astype(np.float32))
    ref = orc.gated_rmsnorm(x.double().numpy(), z.double().numpy(), w.double().numpy(), 1e-6)
    y = gdn.gated_rmsnorm(x.cuda(), z.cuda(), w.cuda(), 1e-6, out_dtype=yt)
    torch.cuda.synchronize()
    _check(y, ref, yt == torch.bfloat16)


def test_standalone_in_place_and_zero_rows(gdn):
    r = np.random.default_rng(9)
    x = torch.from_numpy(r.standard_normal((5, 3, 128)).astype(np.float32))
    x[1, 2] = 0.0
    z = torch.from_numpy(r.standard_normal((5, 3, 128)).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy(r.uniform(0.5, 1.5, 128).astype(np.float32))
    ref = orc.gated_rmsnorm(x.double().numpy(), z.double().numpy(), w.double().numpy(), 1e-6)
    xd = x.cuda()
    gdn.gated_rmsnorm(xd, z.cuda(), w.cuda(), 1e-6, y=xd)
    torch.cuda.synchronize()
    _check(xd, ref, False)
    assert torch.all(xd[1, 2] == 0)


def _gated_case(gdn, B, out_dtype, gates="config", seed=61):
    w = workload("batched_verify", B=B, seed=seed)
    x = make_inputs(w, gates=gates)
    n = make_norm_inputs(w)
    L = x["accept_len"].numpy().copy()
    L[0] = 0
    o_ref, S_ref, _ = oracle_verify(x, L)
    y_ref = orc.gated_rmsnorm(o_ref, n["norm_z"].double().numpy(), n["norm_w"].double().numpy(), 1e-6)
    xd = to_dev(x)
    state = xd["S0"].clone()
    Ld = torch.as_tensor(L).cuda()
    o = gdn.verify_step_gated(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"], state,
                              state, Ld, n["norm_z"].cuda(), n["norm_w"].cuda(), 1e-6, out_dtype=out_dtype)
    torch.cuda.synchronize()
    tol = TOL_BF16_OUT if out_dtype == torch.bfloat16 else TOL
    assert rel_err(o, y_ref) <= tol, rel_err(o, y_ref)
    assert rel_err(state, S_ref) <= TOL


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_verify_gated_tensor_core_kernel(gdn, out_dtype):
    _gated_case(gdn, 64, out_dtype)            # B * H_v = 3072: the fused tensor-core kernel


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_verify_gated_composed_path(gdn, out_dtype):
    _gated_case(gdn, 2, out_dtype)             # 96 heads: mixer, then the standalone pass


def test_verify_gated_gentle_gates(gdn):
    _gated_case(gdn, 64, torch.float32, gates="gentle", seed=62)


def test_verify_gated_two_phase_stash_unaffected(gdn):
    # two-phase: outputs normalised, stash identical to the plain call's, state untouched
    w = workload("batched_verify", B=64, seed=63)
    x, n = make_inputs(w), make_norm_inputs(w)
    xd = to_dev(x)
    nb = gdn.stash_bytes(w.B, w.T, w.H_k, w.H_v, w.d_k, w.d_v) // 4
    s1 = torch.zeros(nb, device="cuda")
    s2 = torch.zeros(nb, device="cuda")
    state = xd["S0"].clone()
    gdn.verify_step(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"], state, None, None,
                    stash=s1)
    o = gdn.verify_step_gated(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"], state,
                              None, None, n["norm_z"].cuda(), n["norm_w"].cuda(), 1e-6, stash=s2)
    torch.cuda.synchronize()
    assert torch.equal(s1, s2) and torch.equal(state, xd["S0"])
    o_ref, _, _ = oracle_verify(x, None)
    y_ref = orc.gated_rmsnorm(o_ref, n["norm_z"].double().numpy(), n["norm_w"].double().numpy(), 1e-6)
    assert rel_err(o, y_ref) <= TOL
