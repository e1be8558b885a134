"""Pins for the oracle's acceptance of a verify block (oracle_accept): planted greedy outcomes,
the tie rule, the sampled acceptance rule against SciPy's softmax at both sides of the p / q
threshold, the bonus draw against NumPy's cumulative sum, the temperature's scale property,
and the theorem that makes speculative sampling exact (the emitted token is distributed as p
whatever q is), checked statistically."""
import numpy as np
import pytest
from scipy.special import softmax

from oracle import gdn_oracle as orc


def test_greedy_planted_outcomes():
    r = np.random.default_rng(1)
    B, T, V = 4, 8, 300
    target = r.standard_normal((B, T, V))
    tokens = r.integers(0, V, (B, T)).astype(np.int32)
    plan = [0, 3, 7, 5]                   # surviving drafts per sequence
    nxt = [11, 22, 33, 44]
    for b, n in enumerate(plan):
        for t in range(n):
            target[b, t, tokens[b, t + 1]] = 10.0
        if n < T - 1:
            target[b, n, tokens[b, n + 1]] = -10.0
        if tokens[b, min(n + 1, T - 1)] == nxt[b]:
            nxt[b] += 1
        target[b, n, nxt[b]] = 12.0
    L, nt, _, _ = orc.accept(target, tokens)
    assert list(L) == [n + 1 for n in plan]
    assert list(nt) == nxt


def test_greedy_ties_take_the_lowest_index():
    target = np.zeros((1, 2, 6))
    target[0, 0, [2, 4]] = 5.0
    target[0, 1, [1, 3]] = 7.0
    L, nt, _, _ = orc.accept(target, np.array([[0, 4]], np.int32))
    assert L[0] == 1 and nt[0] == 2          # the draft 4 ties the maximum but 2 comes first
    L, nt, _, _ = orc.accept(target, np.array([[0, 2]], np.int32))
    assert L[0] == 2 and nt[0] == 1


def test_sampled_rule_at_the_threshold():
    r = np.random.default_rng(2)
    B, T, V = 6, 2, 40
    target, draft = r.standard_normal((B, T, V)), r.standard_normal((B, T - 1, V))
    tokens = r.integers(0, V, (B, T)).astype(np.int32)
    p = softmax(target[:, 0], axis=-1)[np.arange(B), tokens[:, 1]]
    q = softmax(draft[:, 0], axis=-1)[np.arange(B), tokens[:, 1]]
    ratio = p / q
    for side, expect in ((1 - 1e-9, True), (1 + 1e-9, False)):
        u = np.full((B, T), 0.5)
        u[:, 1] = np.minimum(ratio * side, 0.999999)
        L, _, pd, qd = orc.accept(target, tokens, draft, u, sampled=True)
        np.testing.assert_allclose(pd[:, 0], p, rtol=1e-12)
        np.testing.assert_allclose(qd[:, 0], q, rtol=1e-12)
        for b in range(B):
            accepted = L[b] == 2
            if ratio[b] >= 1.0:
                assert accepted                   # min(1, p / q) = 1 accepts every u < 1
            else:
                assert accepted == expect


def test_sampled_identical_models_accept_all_and_draw_the_bonus_from_p():
    r = np.random.default_rng(3)
    B, T, V = 5, 8, 64
    logits = r.standard_normal((B, T, V))
    tokens = r.integers(0, V, (B, T)).astype(np.int32)
    u = r.random((B, T))
    L, nt, _, _ = orc.accept(logits, tokens, logits[:, :T - 1], u, sampled=True)
    assert np.all(L == T)
    for b in range(B):
        cdf = np.cumsum(softmax(logits[b, T - 1]))
        assert nt[b] == np.searchsorted(cdf, u[b, 0] * cdf[-1], side="right")


def test_temperature_scales_logits():
    r = np.random.default_rng(4)
    B, T, V = 8, 4, 30
    target, draft = r.standard_normal((B, T, V)), r.standard_normal((B, T - 1, V))
    tokens = r.integers(0, V, (B, T)).astype(np.int32)
    u = r.random((B, T))
    a = orc.accept(target, tokens, draft, u, tau=0.5, sampled=True)
    b = orc.accept(2.0 * target, tokens, 2.0 * draft, u, tau=1.0, sampled=True)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_emitted_token_is_distributed_as_the_target():
    # one draft per block (T = 2): the drafted token d ~ q, then d if accepted, else the
    # correction; over many blocks the emitted token's frequencies must match p.
    r = np.random.default_rng(5)
    N, V = 200_000, 5
    tl = np.log(np.array([0.4, 0.25, 0.2, 0.1, 0.05]))
    dl = np.log(np.array([0.1, 0.1, 0.5, 0.2, 0.1]))
    p, q = softmax(tl), softmax(dl)
    d = r.choice(V, size=N, p=q)
    tokens = np.stack([np.zeros(N, np.int64), d], axis=1).astype(np.int32)
    target = np.broadcast_to(tl, (N, 2, V)).copy()
    draft = np.broadcast_to(dl, (N, 1, V)).copy()
    u = r.random((N, 2))
    L, nt, _, _ = orc.accept(target, tokens, draft, u, sampled=True)
    emitted = np.where(L == 2, d, nt)
    freq = np.bincount(emitted, minlength=V) / N
    sigma = np.sqrt(p * (1 - p) / N)
    assert np.all(np.abs(freq - p) < 5 * sigma), (freq, p)
    # and the acceptance rate is the overlap sum_j min(p_j, q_j)
    rate = np.mean(L == 2)
    overlap = np.minimum(p, q).sum()
    assert abs(rate - overlap) < 5 * np.sqrt(overlap * (1 - overlap) / N)


@pytest.mark.parametrize("sampled", [False, True])
def test_only_the_leading_run_survives(sampled):
    # drafts 1, 3, 4 would survive on their own, draft 2 does not: one draft is accepted
    V, T = 50, 5
    tokens = np.array([[0, 7, 8, 9, 10]], np.int32)
    target = np.zeros((1, T, V))
    for t in (0, 2, 3):
        target[0, t, tokens[0, t + 1]] = 20.0
    target[0, 1, 30] = 20.0                    # row 1 prefers 30, not the draft 8
    draft = target[:, :T - 1].copy()
    draft[0, 1, :] = 0.0
    draft[0, 1, tokens[0, 2]] = 20.0           # the drafter was sure of 8; the target was not
    u = np.full((1, T), 0.5)
    L, nt, _, _ = orc.accept(target, tokens, draft if sampled else None, u if sampled else None,
                             sampled=sampled)
    assert L[0] == 2 and nt[0] == 30
