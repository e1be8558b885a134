"""Pins for the fp64 CPU oracle: closed forms, invariants, special cases and brute force.

Each test checks the oracle against something other than itself: a value worked out by
hand, an identity the gated delta rule fixes, a textbook special case, or the literal
d x d matrix form on tiny heads. The rule is the Gated DeltaNet update
S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t, with the
state committed at the accepted prefix of a 7 + 1 verify block (source pages:
"Lithos-metal: Qwen3.8-27B on 40-core M5 Max", table "GDN mixer" and the runtime
paragraph; "Qwen 3.8 27B mac m5: 200 tok/s, audited", DSpark section).
"""
import math

import numpy as np
import pytest

from oracle import gdn_oracle as orc
from oracle.brute import brute_recurrence


def rel_err(x, ref):
    x, ref = np.asarray(x), np.asarray(ref)
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-300))


def rand_case(rng, B=1, T=8, Hk=1, Hv=2, dk=16, dv=16, state_std=0.1, gentle=False):
    q = rng.standard_normal((B, T, Hk, dk))
    k = rng.standard_normal((B, T, Hk, dk))
    v = rng.standard_normal((B, T, Hv, dv))
    a = rng.standard_normal((B, T, Hv)) - (6.0 if gentle else 0.0)
    b = rng.standard_normal((B, T, Hv))
    A_log = rng.uniform(0.0, math.log(16.0), Hv)
    dt_bias = np.zeros(Hv)
    S0 = rng.standard_normal((B, Hv, dv, dk)) * state_std
    return q, k, v, a, b, A_log, dt_bias, S0


# ---------------------------------------------------------------- gates and norm


def test_gates_closed_forms():
    # A_log = 0, a = 0: log_alpha = -1 * softplus(0) = -ln 2, so alpha = 1/2.
    # A_log = ln 2, a = 0: log_alpha = -2 ln 2, alpha = 1/4.
    # a = ln(e - 1): softplus = ln(1 + e - 1) = 1, so log_alpha = -exp(A_log).
    # b = 0: beta = 1/2; b = ln 3: beta = 1 / (1 + 1/3) = 3/4.
    a = np.array([[0.0, 0.0, math.log(math.e - 1.0)]])
    b = np.array([[0.0, math.log(3.0), -math.log(3.0)]])
    A_log = np.array([0.0, math.log(2.0), 0.7])
    la, be = orc.gates(a, b, A_log, np.zeros(3))
    assert np.exp(la[0, 0]) == pytest.approx(0.5, abs=1e-15)
    assert np.exp(la[0, 1]) == pytest.approx(0.25, abs=1e-15)
    assert la[0, 2] == pytest.approx(-math.exp(0.7), rel=1e-14)
    assert be[0, 0] == pytest.approx(0.5, abs=1e-16)
    assert be[0, 1] == pytest.approx(0.75, abs=1e-15)
    assert be[0, 2] == pytest.approx(0.25, abs=1e-15)


def test_gates_softplus_identity_and_bias():
    # softplus(x) - softplus(-x) = x, so log_alpha(x) - log_alpha(-x) = -exp(A_log) x;
    # dt_bias only shifts the argument of softplus; large x gives softplus(x) ~ x.
    x = np.linspace(-30, 30, 61)[None, :]
    A_log = np.full(61, 0.3)
    la_p, _ = orc.gates(x, np.zeros_like(x), A_log, np.zeros(61))
    la_m, _ = orc.gates(-x, np.zeros_like(x), A_log, np.zeros(61))
    np.testing.assert_allclose(la_p - la_m, -math.exp(0.3) * x, rtol=1e-12, atol=1e-12)
    la_b, _ = orc.gates(x - 1.5, np.zeros_like(x), A_log, np.full(61, 1.5))
    np.testing.assert_allclose(la_b, la_p, rtol=1e-14, atol=0)
    la_big, _ = orc.gates(np.array([[40.0]]), np.zeros((1, 1)), np.array([0.0]), np.zeros(1))
    assert la_big[0, 0] == pytest.approx(-40.0, rel=1e-15)


def test_gates_saturate_exactly():
    # a = -1e4: softplus underflows to exactly 0, so alpha = exp(-0) = 1;
    # b = -1e4: beta = 1 / (1 + inf) = 0; b = +1e4: beta = 1.
    la, be = orc.gates(np.array([[-1e4, -1e4]]), np.array([[-1e4, 1e4]]),
                       np.array([2.0, 2.0]), np.zeros(2))
    assert np.exp(la[0, 0]) == 1.0 and np.exp(la[0, 1]) == 1.0
    assert be[0, 0] == 0.0 and be[0, 1] == 1.0


def test_l2norm_closed_forms():
    y = orc.l2norm(np.array([[3.0, 4.0]]), eps=0.0)
    np.testing.assert_allclose(y, [[0.6, 0.8]], rtol=0, atol=4e-16)
    y = orc.l2norm(np.array([[3.0, 4.0]]), eps=11.0)          # sqrt(25 + 11) = 6
    np.testing.assert_allclose(y, [[0.5, 4.0 / 6.0]], rtol=0, atol=4e-16)
    y = orc.l2norm(np.array([[3.0, 4.0]]), eps=0.0, scale=0.25)
    np.testing.assert_allclose(y, [[0.15, 0.2]], rtol=0, atol=4e-16)
    x = np.random.default_rng(0).standard_normal((50, 128))
    n = np.linalg.norm(orc.l2norm(x, eps=0.0), axis=1)
    np.testing.assert_allclose(n, 1.0, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- the recurrence


def test_scalar_head_worked_example():
    # d = 1, k = q = 1 with eps = 0 gives khat = qhat = 1, and with A_log = a = b = 0
    # both gates are 1/2. The rule becomes the scalar recursion
    #   S_t = alpha (1 - beta) S_{t-1} + beta v_t = S_{t-1} / 4 + v_t / 2,  o_t = S_t.
    # From S_0 = 1 and v = (2, 4, 8), by hand:
    #   S_1 = 1/4 + 1 = 1.25, S_2 = 1.25/4 + 2 = 2.3125, S_3 = 2.3125/4 + 4 = 4.578125.
    one = np.ones((1, 3, 1, 1))
    v = np.array([2.0, 4.0, 8.0]).reshape(1, 3, 1, 1)
    z = np.zeros((1, 3, 1))
    o, Sc, bad = orc.verify(one, one, v, z, z, np.zeros(1), np.zeros(1), np.ones((1, 1, 1, 1)),
                            None, l2_eps=0.0)
    np.testing.assert_allclose(o.ravel(), [1.25, 2.3125, 4.578125], rtol=1e-14)
    assert Sc.ravel()[0] == pytest.approx(4.578125, rel=1e-14)
    assert bad[0] == 0
    # commit after the first two tokens only
    o, Sc, _ = orc.verify(one, one, v, z, z, np.zeros(1), np.zeros(1), np.ones((1, 1, 1, 1)),
                          np.array([2]), l2_eps=0.0)
    assert Sc.ravel()[0] == pytest.approx(2.3125, rel=1e-14)


def test_identity_beta0_alpha1_full_pipeline():
    # a = -1e4 (alpha = 1 exactly) and b = -1e4 (beta = 0 exactly): the state never moves.
    rng = np.random.default_rng(1)
    q, k, v, a, b, A_log, dt, S0 = rand_case(rng, B=2, T=8, Hk=2, Hv=4)
    a[:] = -1e4
    b[:] = -1e4
    o, Sc, _ = orc.verify(q, k, v, a, b, A_log, dt, S0, np.array([8, 5]))
    assert np.array_equal(Sc, S0)
    # and each output is the untouched state applied to the query
    qh = orc.l2norm(q)
    for h in range(4):
        np.testing.assert_allclose(o[:, :, h], np.einsum("bij,btj->bti", S0[:, h], qh[:, :, h // 2]),
                                   rtol=0, atol=1e-14)


def test_write_then_read():
    # alpha = beta = 1 and a unit key: S_t khat_t = v_t right after the write, so with
    # q_t = k_t the output o_t = S_t qhat_t equals v_t. A rule that read S_{t-1} for the
    # output, or had the sign of the beta term flipped, would fail here.
    rng = np.random.default_rng(2)
    B, T, H, d = 2, 8, 3, 16
    k = rng.standard_normal((B, T, 1, d))
    v = rng.standard_normal((B, T, H, d))
    S0 = rng.standard_normal((B, H, d, d)) * 0.3
    ones = np.ones((B, T, H))
    kh = orc.l2norm(k, eps=0.0)
    o, Sc, _ = orc.recurrence(kh, kh, v, ones, ones, S0, None)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)
    np.testing.assert_allclose(np.einsum("bhij,bj->bhi", Sc, kh[:, -1, 0]), v[:, -1], atol=1e-12)


def test_orthonormal_keys_recall_every_pair():
    # alpha = beta = 1, orthonormal keys k_1..k_T: every write is a projection onto a fresh
    # direction, so S_T = S_0 (I - sum k k^T) + sum v_t k_t^T and S_T k_i = v_i for all i.
    rng = np.random.default_rng(3)
    d, T = 16, 8
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = Qm[:, :T].T                                     # T orthonormal rows
    kh = keys.reshape(1, T, 1, d)
    v = rng.standard_normal((1, T, 1, d))
    S0 = rng.standard_normal((1, 1, d, d))
    ones = np.ones((1, T, 1))
    _, Sc, _ = orc.recurrence(kh, kh, v, ones, ones, S0, None)
    P = keys.T @ keys
    expect = S0[0, 0] @ (np.eye(d) - P) + v[0, :, 0].T @ keys
    np.testing.assert_allclose(Sc[0, 0], expect, atol=1e-12)
    np.testing.assert_allclose(keys @ Sc[0, 0].T, v[0, :, 0], atol=1e-12)


def test_pure_decay_closed_form():
    # beta = 0: S_L = (prod_{t<=L} alpha_t) S_0 and o_t = (prod_{m<=t} alpha_m) S_0 qhat_t.
    rng = np.random.default_rng(4)
    B, T, H, d = 1, 8, 2, 16
    q, k, v, *_ = rand_case(rng, B=B, T=T, Hk=1, Hv=H, dk=d, dv=d)
    alpha = rng.uniform(0.2, 1.0, (B, T, H))
    beta = np.zeros((B, T, H))
    S0 = rng.standard_normal((B, H, d, d))
    qh, kh = orc.l2norm(q), orc.l2norm(k)
    for L in range(T + 1):
        o, Sc, _ = orc.recurrence(qh, kh, v, alpha, beta, S0, np.array([L]))
        for h in range(H):
            np.testing.assert_allclose(Sc[0, h], np.prod(alpha[0, :L, h]) * S0[0, h], rtol=1e-13)
    for t in range(T):
        for h in range(H):
            np.testing.assert_allclose(o[0, t, h], np.prod(alpha[0, :t + 1, h]) * S0[0, h] @ qh[0, t, 0],
                                       rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("gentle", [False, True])
def test_brute_force_matrix_form(gentle):
    # Literal d x d products (I - beta k k^T) against the oracle's rank-1 expansion,
    # on 2 sequences, 2 key heads shared by 4 value heads, d = 16, T = 8.
    rng = np.random.default_rng(5 + gentle)
    q, k, v, a, b, A_log, dt, S0 = rand_case(rng, B=2, T=8, Hk=2, Hv=4, gentle=gentle)
    la, be = orc.gates(a, b, A_log, dt)
    qh, kh = orc.l2norm(q, scale=0.7), orc.l2norm(k)
    L = np.array([3, 8])
    o, Sc, _ = orc.recurrence(qh, kh, v, np.exp(la), be, S0, L)
    ob, Sb = brute_recurrence(qh, kh, v, np.exp(la), be, S0, L)
    assert rel_err(o, ob) < 1e-12
    assert rel_err(Sc, Sb) < 1e-12
    o2, Sc2, _ = orc.verify(q, k, v, a, b, A_log, dt, S0, L, scale=0.7)
    assert rel_err(o2, ob) < 1e-12 and rel_err(Sc2, Sb) < 1e-12


def test_brute_force_rectangular_head():
    # d_k != d_v: S is d_v x d_k; a transposed state would not even have the right shape
    # in the brute-force product S @ (I - beta k k^T).
    rng = np.random.default_rng(7)
    q, k, v, a, b, A_log, dt, S0 = rand_case(rng, B=1, T=5, Hk=1, Hv=2, dk=8, dv=12)
    la, be = orc.gates(a, b, A_log, dt)
    qh, kh = orc.l2norm(q), orc.l2norm(k)
    o, Sc, _ = orc.recurrence(qh, kh, v, np.exp(la), be, S0, None)
    ob, Sb = brute_recurrence(qh, kh, v, np.exp(la), be, S0, None)
    assert rel_err(o, ob) < 1e-12 and rel_err(Sc, Sb) < 1e-12


def test_commit_equals_prefix_recurrence_and_rollback_is_exact():
    rng = np.random.default_rng(8)
    q, k, v, a, b, A_log, dt, S0 = rand_case(rng, B=1, T=8, Hk=1, Hv=3, gentle=True)
    for L in range(9):
        o, Sc, bad = orc.verify(q, k, v, a, b, A_log, dt, S0, np.array([L]))
        assert bad[0] == 0
        if L == 0:
            assert np.array_equal(Sc, S0)                      # rollback: bit-identical
            continue
        _, Sp, _ = orc.verify(q[:, :L], k[:, :L], v[:, :L], a[:, :L], b[:, :L], A_log, dt, S0,
                              None)
        assert np.array_equal(Sc, Sp)
        # outputs do not depend on the commit point
        o8, _, _ = orc.verify(q, k, v, a, b, A_log, dt, S0, None)
        assert np.array_equal(o, o8)


def test_out_of_range_accept_len_commits_nothing():
    rng = np.random.default_rng(9)
    q, k, v, a, b, A_log, dt, S0 = rand_case(rng, B=3, T=8, Hk=1, Hv=2)
    o, Sc, bad = orc.verify(q, k, v, a, b, A_log, dt, S0, np.array([-1, 9, 4]))
    assert list(bad) == [1, 1, 0]
    assert np.array_equal(Sc[0], S0[0]) and np.array_equal(Sc[1], S0[1])
    assert not np.array_equal(Sc[2], S0[2])


def test_gqa_contiguous_groups():
    # value head h reads key head h // (H_v / H_k): with H_k = 2, H_v = 4, heads 0,1 use
    # key head 0 and heads 2,3 use key head 1. Each head is recomputed alone with the
    # key head it should see.
    rng = np.random.default_rng(10)
    q, k, v, a, b, A_log, dt, S0 = rand_case(rng, B=1, T=6, Hk=2, Hv=4)
    o, Sc, _ = orc.verify(q, k, v, a, b, A_log, dt, S0, None)
    for h in range(4):
        g = h // 2
        o1, S1, _ = orc.verify(q[:, :, g:g + 1], k[:, :, g:g + 1], v[:, :, h:h + 1],
                               a[:, :, h:h + 1], b[:, :, h:h + 1], A_log[h:h + 1], dt[h:h + 1],
                               S0[:, h:h + 1], None)
        assert np.array_equal(o[:, :, h:h + 1], o1) and np.array_equal(Sc[:, h:h + 1], S1)


def test_output_scale_is_linear():
    rng = np.random.default_rng(11)
    q, k, v, a, b, A_log, dt, S0 = rand_case(rng, B=1, T=8, Hk=1, Hv=2)
    o1, S1, _ = orc.verify(q, k, v, a, b, A_log, dt, S0, None, scale=1.0)
    o2, S2, _ = orc.verify(q, k, v, a, b, A_log, dt, S0, None, scale=0.125)
    np.testing.assert_allclose(o2, 0.125 * o1, rtol=1e-13, atol=1e-16)
    assert np.array_equal(S1, S2)


# ---------------------------------------------------------------- chunked form


@pytest.mark.parametrize("T,C,gentle,zero_state", [
    (256, 16, True, False), (256, 64, True, False), (256, 64, False, False),
    (100, 16, True, False), (100, 64, True, True), (7, 16, False, False), (1, 64, True, False)])
def test_chunked_equals_recurrent(T, C, gentle, zero_state):
    rng = np.random.default_rng(100 + T + C)
    q, k, v, a, b, A_log, dt, S0 = rand_case(rng, B=1, T=T, Hk=1, Hv=2, dk=16, dv=16,
                                             gentle=gentle)
    if zero_state:
        S0 = np.zeros_like(S0)
    la, be = orc.gates(a, b, A_log, dt)
    qh, kh = orc.l2norm(q), orc.l2norm(k)
    o_r, S_r, _ = orc.recurrence(qh, kh, v, np.exp(la), be, S0, None)
    o_c, S_c = orc.chunked(qh, kh, v, la, be, None if zero_state else S0, C)
    assert rel_err(o_c, o_r) < 1e-10
    assert rel_err(S_c, S_r) < 1e-10


def test_chunked_survives_total_decay_underflow():
    # Strong gates: cumulative log-decay in a 64-chunk goes far below -745, where exp()
    # of it underflows in fp64; only differences G_t - G_s may be exponentiated.
    rng = np.random.default_rng(12)
    q, k, v, a, b, A_log, dt, S0 = rand_case(rng, B=1, T=128, Hk=1, Hv=2)
    a = a + 3.0
    A_log[:] = math.log(16.0)
    la, be = orc.gates(a, b, A_log, dt)
    assert la.sum(axis=1).min() < -2000
    qh, kh = orc.l2norm(q), orc.l2norm(k)
    o_r, S_r, _ = orc.recurrence(qh, kh, v, np.exp(la), be, S0, None)
    o_c, S_c = orc.chunked(qh, kh, v, la, be, S0, 64)
    assert np.isfinite(o_c).all() and np.isfinite(S_c).all()
    assert rel_err(o_c, o_r) < 1e-10 and rel_err(S_c, S_r) < 1e-10
