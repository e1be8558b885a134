"""Brute-force NumPy form of the gated delta rule, for tiny heads only.

TEST INFRASTRUCTURE: used by the tests to pin the C oracle.

Unlike gdn_oracle.c, which expands S (I - beta k k^T) into a rank-1 update,
this forms the d_k x d_k matrix (I - beta_t khat_t khat_t^T) explicitly and
multiplies by it, token by token, exactly as the rule is written (Gated
DeltaNet update, source page "Lithos-metal: Qwen3.8-27B on 40-core M5 Max",
table "GDN mixer"; output o_t = S_t qhat_t; commit at the accepted prefix,
same page, runtime paragraph). Pure Python loops over (b, h, t): keep d <= 32.
"""
import numpy as np


def brute_recurrence(qhat, khat, v, alpha, beta, S0, accept_len=None):
    """qhat, khat: [B,T,Hk,dk]; v: [B,T,Hv,dv]; alpha, beta: [B,T,Hv]; S0: [B,Hv,dv,dk].

    Returns (o [B,T,Hv,dv], S_commit [B,Hv,dv,dk]).
    """
    qhat, khat, v, alpha, beta, S0 = (np.asarray(x, dtype=np.float64)
                                      for x in (qhat, khat, v, alpha, beta, S0))
    B, T, Hk, dk = khat.shape
    Hv, dv = v.shape[2], v.shape[3]
    G = Hv // Hk
    o = np.zeros((B, T, Hv, dv))
    Sc = np.zeros((B, Hv, dv, dk))
    eye = np.eye(dk)
    for b in range(B):
        L = T if accept_len is None else int(accept_len[b])
        for h in range(Hv):
            g = h // G
            S = S0[b, h].copy()
            if L == 0:
                Sc[b, h] = S
            for t in range(T):
                k = khat[b, t, g]
                M = eye - beta[b, t, h] * np.outer(k, k)
                S = alpha[b, t, h] * (S @ M) + beta[b, t, h] * np.outer(v[b, t, h], k)
                o[b, t, h] = S @ qhat[b, t, g]
                if t + 1 == L:
                    Sc[b, h] = S
    return o, Sc
