"""GPU parity for gdn_accept (device-side acceptance of verify blocks) against the fp64
oracle, through the C ABI.

Greedy acceptance and its next token are decided by exact comparisons of the stored logits:
bit-exact against the oracle. Sampled acceptance decides u * q < p in fp32 on the GPU and in
fp64 in the oracle, so both are compared where the decision is not within 1e-3 (relative) of
its threshold; a sequence whose deciding comparison is that close is skipped (and counted).
The drawn token can differ where the cumulative mass sits near u * total, so it is checked
for validity against the fp64 residual (its cumulative interval contains u * total within
1e-4 of the total, and its weight is positive), and for equality with the oracle in all but
a few sequences. A statistical check runs the theorem that makes speculative sampling exact
on the GPU: the emitted token is distributed as p."""
import numpy as np
import pytest
import torch
from scipy.special import softmax

from gated_deltanet_mixer_verify_b200.inputs import make_accept_inputs, workload
from oracle import gdn_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn(cuda_device):
    from gated_deltanet_mixer_verify_b200 import build, gdn as g
    build.build()
    return g


def _f64(t):
    return t.double().numpy()


def _run(gdn, x, sampled, tau=1.0):
    d = {k: v.cuda() for k, v in x.items()}
    L, nt = gdn.accept(d["target"], d["tokens"], d["draft"] if sampled else None,
                       d["uniforms"] if sampled else None, temperature=tau)
    torch.cuda.synchronize()
    return L.cpu().numpy(), nt.cpu().numpy()


@pytest.mark.parametrize("B,T,V,dtype", [(64, 8, 151936, "bf16"), (5, 8, 1000, "f32"), (7, 3, 4104, "bf16"),
                                         (3, 1, 64, "f32")])
def test_greedy_bit_exact(gdn, B, T, V, dtype):
    w = workload("batched_verify", B=B, T=T, seed=81)
    x = make_accept_inputs(w, V=V, dtype=dtype)
    L, nt = _run(gdn, x, sampled=False)
    Lr, ntr, _, _ = orc.accept(_f64(x["target"]), x["tokens"].numpy())
    np.testing.assert_array_equal(L, Lr)
    np.testing.assert_array_equal(nt, ntr)
    if B * T > 8:
        assert len(set(Lr.tolist())) > 2          # a spread of accept counts was exercised


def test_greedy_ties_take_the_lowest_index(gdn):
    V = 4096
    target = torch.zeros((2, 3, V))
    target[0, 0, [4000, 17]] = 3.0                  # draft 4000 ties the maximum: rejected (17 first)
    target[1, 0, [9, 2048]] = 3.0                   # draft 9 is the first maximum: accepted
    target[1, 1, [300, 3000]] = 5.0
    tokens = torch.tensor([[1, 4000, 2], [1, 9, 5]], dtype=torch.int32)
    L, nt = gdn.accept(target.cuda(), tokens.cuda())
    torch.cuda.synchronize()
    assert L.tolist() == [1, 2] and nt.tolist() == [17, 300]


def _residual_cdf(x, b, n, tau):
    T = x["target"].shape[1]
    p = softmax(_f64(x["target"][b, n]) / tau)
    if n < T - 1:
        r = np.maximum(p - softmax(_f64(x["draft"][b, n]) / tau), 0.0)
        if r.sum() > 0:
            return r
    return p


def _check_sampled(gdn, x, tau, max_skipped, max_token_mismatch):
    L, nt = _run(gdn, x, sampled=True, tau=tau)
    f = {k: _f64(v) for k, v in x.items() if k != "tokens"}
    tokens = x["tokens"].numpy()
    Lr, ntr, pd, qd = orc.accept(f["target"], tokens, f["draft"], f["uniforms"], tau=tau, sampled=True)
    u = f["uniforms"]
    B, T = tokens.shape
    skipped = mism = 0
    for b in range(B):
        # the decisions up to and including the first rejection (or all of them)
        close = False
        for t in range(min(Lr[b], T - 1)):
            p, q = pd[b, t], qd[b, t]
            if abs(u[b, t + 1] * q - p) <= 1e-3 * max(p, 1e-30):
                close = True
        if close:
            skipped += 1
            continue
        assert L[b] == Lr[b], (b, L[b], Lr[b])
        r = _residual_cdf(x, b, L[b] - 1, tau)
        cdf = np.cumsum(r)
        tot = cdf[-1]
        j = nt[b]
        target = u[b, 0] * tot
        lo = cdf[j - 1] if j > 0 else 0.0
        assert r[j] > 0 and lo - 1e-4 * tot <= target <= cdf[j] + 1e-4 * tot, (b, j, ntr[b])
        mism += int(j != ntr[b])
    assert skipped <= max_skipped and mism <= max_token_mismatch, (skipped, mism)
    return L


def test_sampled_full_vocabulary(gdn):
    w = workload("batched_verify", B=64, T=8, seed=82)
    x = make_accept_inputs(w)                                   # V = 151,936, bf16
    L = _check_sampled(gdn, x, 1.0, max_skipped=3, max_token_mismatch=2)
    assert len(set(L.tolist())) > 2


def test_sampled_temperature_fp32_many_sequences(gdn):
    w = workload("batched_verify", B=256, T=8, seed=83)
    x = make_accept_inputs(w, V=1024, dtype="f32", plant=0.6)
    _check_sampled(gdn, x, 0.7, max_skipped=8, max_token_mismatch=4)


def test_sampled_all_accepted_draws_the_bonus(gdn):
    w = workload("batched_verify", B=32, T=8, seed=84)
    x = make_accept_inputs(w, V=2048, dtype="f32")
    x["draft"] = x["target"][:, :7].clone()                    # p == q: every draft survives
    L = _check_sampled(gdn, x, 1.0, max_skipped=0, max_token_mismatch=1)
    assert np.all(L == 8)


def test_emitted_token_is_distributed_as_the_target(gdn):
    # the theorem behind exact speculative sampling, on the GPU: one draft per block, drafted
    # from q; the emitted token (the draft if accepted, else the correction) follows p.
    r = np.random.default_rng(85)
    N, V = 65536, 8
    pl = np.log(np.array([0.3, 0.2, 0.15, 0.1, 0.1, 0.08, 0.05, 0.02]))
    ql = np.log(np.array([0.05, 0.1, 0.3, 0.2, 0.1, 0.1, 0.1, 0.05]))
    p = softmax(pl)
    d = r.choice(V, size=N, p=softmax(ql))
    tokens = torch.from_numpy(np.stack([np.zeros(N, np.int64), d], 1).astype(np.int32))
    target = torch.from_numpy(np.broadcast_to(pl, (N, 2, V)).astype(np.float32).copy())
    draft = torch.from_numpy(np.broadcast_to(ql, (N, 1, V)).astype(np.float32).copy())
    u = torch.from_numpy(r.random((N, 2)).astype(np.float32))
    L, nt = gdn.accept(target.cuda(), tokens.cuda(), draft.cuda(), u.cuda())
    torch.cuda.synchronize()
    emitted = np.where(L.cpu().numpy() == 2, d, nt.cpu().numpy())
    freq = np.bincount(emitted, minlength=V) / N
    assert np.all(np.abs(freq - p) < 5 * np.sqrt(p * (1 - p) / N)), (freq, p)
