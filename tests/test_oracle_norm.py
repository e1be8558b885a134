"""Pins for the oracle's gated RMS normalisation of the mixer output (oracle_gated_rmsnorm),
against PyTorch's own rms_norm and silu (fp64), a worked example with a closed form, and the
invariances the definition implies."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import gdn_oracle as orc


@pytest.mark.parametrize("eps", [1e-6, 0.3])
def test_matches_torch_rms_norm_and_silu(eps):
    r = np.random.default_rng(3)
    o = r.standard_normal((5, 3, 16))
    z = r.standard_normal((5, 3, 16)) * 2
    w = r.uniform(0.5, 1.5, 16)
    y = orc.gated_rmsnorm(o, z, w, eps)
    ref = F.rms_norm(torch.from_numpy(o), (16,), weight=torch.from_numpy(w), eps=eps) * F.silu(torch.from_numpy(z))
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-13, atol=1e-15)


def test_worked_example():
    # o = (3, 4, 0, 0): mean square 25/4, rms 2.5; z = ln 3 gives silu = (3/4) ln 3; w = (1, 2, 3, 4)
    o = np.array([[3.0, 4.0, 0.0, 0.0]])
    z = np.full((1, 4), math.log(3.0))
    w = np.array([1.0, 2.0, 3.0, 4.0])
    y = orc.gated_rmsnorm(o, z, w, eps=0.0)
    g = 0.75 * math.log(3.0)
    np.testing.assert_allclose(y[0], [1.2 * g, 1.6 * 2 * g, 0.0, 0.0], rtol=1e-15)


def test_scale_and_sign_invariance():
    r = np.random.default_rng(4)
    o, z, w = r.standard_normal((4, 32)), r.standard_normal((4, 32)), r.standard_normal(32)
    y = orc.gated_rmsnorm(o, z, w, eps=0.0)
    np.testing.assert_allclose(orc.gated_rmsnorm(7.5 * o, z, w, eps=0.0), y, rtol=1e-13)
    np.testing.assert_allclose(orc.gated_rmsnorm(-o, z, w, eps=0.0), -y, rtol=1e-13)
    # with eps > 0 the invariance fails where the rows are small against eps
    y_small = orc.gated_rmsnorm(1e-3 * o, z, w, eps=1e-6)
    assert np.max(np.abs(y_small - y)) > 1e-3


def test_zero_row_and_rows_independent():
    r = np.random.default_rng(5)
    o, z, w = r.standard_normal((3, 8)), r.standard_normal((3, 8)), r.standard_normal(8)
    o[1] = 0.0
    y = orc.gated_rmsnorm(o, z, w, eps=1e-6)
    assert np.all(y[1] == 0.0)
    o2 = o.copy()
    o2[2] *= 10.0
    o2[2, 0] += 1.0
    y2 = orc.gated_rmsnorm(o2, z, w, eps=1e-6)
    np.testing.assert_array_equal(y2[:2], y[:2])
