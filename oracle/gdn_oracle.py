"""ctypes wrapper around the fp64 C oracle (gdn_oracle.c).

TEST INFRASTRUCTURE: imported only by ``tests/``, ``__graft_entry__.smoke()``
and the benchmark's CPU-baseline / reference leg.

The mixer it computes (Gated DeltaNet, verify block of 7 drafts + 1 anchor,
commit / rollback at the accepted prefix) is stated in the header of
gdn_oracle.c; the source pages are "Lithos-metal: Qwen3.8-27B on 40-core M5
Max" (table "GDN mixer"; runtime paragraph on recurrent-state commit/rollback)
and "Qwen 3.8 27B mac m5: 200 tok/s, audited" (sections on fusing layer
mixers and on DSpark verification and rewind).

All arrays are float64 NumPy arrays in the layouts below; nothing here does any
arithmetic of the method itself except via the C library.
"""
import ctypes
import os

import numpy as np

from .build import build_oracle

_lib = None
_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)


def _load():
    global _lib
    if _lib is None:
        # GDN_ORACLE_LIB lets the mutation tests load a deliberately broken copy.
        lib = ctypes.CDLL(os.environ.get("GDN_ORACLE_LIB") or build_oracle())
        lib.oracle_l2norm.argtypes = [ctypes.c_int64, ctypes.c_int, _D, ctypes.c_double,
                                      ctypes.c_double, _D]
        lib.oracle_l2norm.restype = None
        lib.oracle_gates.argtypes = [ctypes.c_int64, ctypes.c_int, _D, _D, _D, _D, _D, _D]
        lib.oracle_gates.restype = None
        lib.oracle_recurrence.argtypes = [ctypes.c_int] * 6 + [_D] * 6 + [_I32, _D, _D, _I32,
                                                                          ctypes.c_int]
        lib.oracle_recurrence.restype = ctypes.c_int
        lib.oracle_verify.argtypes = ([ctypes.c_int] * 6 + [_D] * 8 + [_I32, ctypes.c_double,
                                                                       ctypes.c_double, _D, _D,
                                                                       _I32, ctypes.c_int])
        lib.oracle_verify.restype = ctypes.c_int
        lib.oracle_chunked.argtypes = [ctypes.c_int] * 7 + [_D] * 6 + [_D, _D, ctypes.c_int]
        lib.oracle_chunked.restype = ctypes.c_int
        lib.oracle_short_conv.argtypes = [ctypes.c_int] * 4 + [_D] * 3 + [_I32, _D, _D]
        lib.oracle_short_conv.restype = ctypes.c_int
        lib.oracle_gated_rmsnorm.argtypes = [ctypes.c_int64, ctypes.c_int, _D, _D, _D, ctypes.c_double, _D]
        lib.oracle_gated_rmsnorm.restype = None
        lib.oracle_accept.argtypes = [ctypes.c_int] * 3 + [_D, _D, _I32, _D, ctypes.c_double, ctypes.c_int,
                                                           _I32, _I32, _D, _D]
        lib.oracle_accept.restype = ctypes.c_int
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(x):
    return x.ctypes.data_as(_D) if x is not None else None


def _pi(x):
    return x.ctypes.data_as(_I32) if x is not None else None


def max_threads() -> int:
    """Threads the oracle's OpenMP loops use by default."""
    return int(_load().oracle_max_threads())


def l2norm(x, eps=1e-6, scale=1.0):
    """Rows of x (last axis) scaled to unit L2 norm: scale * x / sqrt(sum x^2 + eps)."""
    x = _f64(x)
    d = x.shape[-1]
    y = np.empty_like(x)
    _load().oracle_l2norm(x.size // d if d else 0, d, _p(x), eps, scale, _p(y))
    return y


def gates(a, b, A_log, dt_bias):
    """(log_alpha, beta) for a, b of shape [..., H_v]; A_log, dt_bias of shape [H_v]."""
    a, b, A_log, dt_bias = _f64(a), _f64(b), _f64(A_log), _f64(dt_bias)
    Hv = a.shape[-1]
    la = np.empty_like(a)
    be = np.empty_like(b)
    _load().oracle_gates(a.size // Hv, Hv, _p(a), _p(b), _p(A_log), _p(dt_bias), _p(la), _p(be))
    return la, be


def recurrence(qhat, khat, v, alpha, beta, S0, accept_len=None, nthreads=0):
    """Per-token recurrence on normalised inputs and given gates.

    qhat, khat: [B, T, H_k, d_k]; v: [B, T, H_v, d_v]; alpha, beta: [B, T, H_v];
    S0: [B, H_v, d_v, d_k]; accept_len: [B] int or None (commit after all T).
    Returns (o [B, T, H_v, d_v], S_commit [B, H_v, d_v, d_k], bad_accept [B]).
    """
    qhat, khat, v, alpha, beta, S0 = map(_f64, (qhat, khat, v, alpha, beta, S0))
    B, T, Hk, dk = khat.shape
    Hv, dv = v.shape[2], v.shape[3]
    o = np.zeros((B, T, Hv, dv))
    Sc = np.zeros((B, Hv, dv, dk))
    bad = np.zeros(B, dtype=np.int32)
    L = None if accept_len is None else np.ascontiguousarray(accept_len, dtype=np.int32)
    rc = _load().oracle_recurrence(B, T, Hk, Hv, dk, dv, _p(qhat), _p(khat), _p(v), _p(alpha),
                                   _p(beta), _p(S0), _pi(L), _p(o), _p(Sc), _pi(bad), nthreads)
    if rc != 0:
        raise ValueError("oracle_recurrence: inconsistent shape")
    return o, Sc, bad


def verify(q, k, v, a, b, A_log, dt_bias, S0, accept_len=None, l2_eps=1e-6, scale=1.0,
           nthreads=0):
    """The whole mixer from raw inputs (normalisation, gates, recurrence, commit).

    q, k: [B, T, H_k, d_k]; v: [B, T, H_v, d_v]; a, b: [B, T, H_v]; A_log, dt_bias: [H_v];
    S0: [B, H_v, d_v, d_k]; accept_len: [B] or None.
    Returns (o, S_commit, bad_accept) as in :func:`recurrence`.
    """
    q, k, v, a, b, A_log, dt_bias, S0 = map(_f64, (q, k, v, a, b, A_log, dt_bias, S0))
    B, T, Hk, dk = k.shape
    Hv, dv = v.shape[2], v.shape[3]
    o = np.zeros((B, T, Hv, dv))
    Sc = np.zeros((B, Hv, dv, dk))
    bad = np.zeros(B, dtype=np.int32)
    L = None if accept_len is None else np.ascontiguousarray(accept_len, dtype=np.int32)
    rc = _load().oracle_verify(B, T, Hk, Hv, dk, dv, _p(q), _p(k), _p(v), _p(a), _p(b),
                               _p(A_log), _p(dt_bias), _p(S0), _pi(L), l2_eps, scale, _p(o),
                               _p(Sc), _pi(bad), nthreads)
    if rc != 0:
        raise ValueError("oracle_verify: inconsistent shape")
    return o, Sc, bad


def chunked(qhat, khat, v, log_alpha, beta, S0, chunk, nthreads=0):
    """Chunked (WY / UT) form on normalised inputs and log-gates.

    S0 may be None (zero initial state). Returns (o, S_final).
    """
    qhat, khat, v, log_alpha, beta = map(_f64, (qhat, khat, v, log_alpha, beta))
    S0 = None if S0 is None else _f64(S0)
    B, T, Hk, dk = khat.shape
    Hv, dv = v.shape[2], v.shape[3]
    o = np.zeros((B, T, Hv, dv))
    Sf = np.zeros((B, Hv, dv, dk))
    rc = _load().oracle_chunked(B, T, Hk, Hv, dk, dv, int(chunk), _p(qhat), _p(khat), _p(v),
                                _p(log_alpha), _p(beta), _p(S0), _p(o), _p(Sf), nthreads)
    if rc != 0:
        raise ValueError("oracle_chunked: inconsistent shape or chunk")
    return o, Sf


def prefill(q, k, v, a, b, A_log, dt_bias, S0=None, l2_eps=1e-6, scale=1.0, nthreads=0):
    """Long-prompt reference: the per-token recurrence over all T tokens, state after T.

    S0 None means a zero initial state. Returns (o, S_final).
    """
    k = _f64(k)
    B, T, Hk, dk = k.shape
    Hv, dv = v.shape[2], v.shape[3]
    if S0 is None:
        S0 = np.zeros((B, Hv, dv, dk))
    o, Sf, _ = verify(q, k, v, a, b, A_log, dt_bias, S0, None, l2_eps, scale, nthreads)
    return o, Sf


def short_conv_channels(x, w, hist, accept_len=None, write_history=True):
    """Causal short convolution per channel with its rewound history (oracle_short_conv).

    x: [B, T, C]; w: [C, K]; hist: [B, K-1, C] (oldest first); accept_len: [B] or None (all T).
    Returns (y [B, T, C], new history [B, K-1, C] or None, number of out-of-range counts).
    """
    x, w, hist = _f64(x), _f64(w), _f64(hist)
    B, T, C = x.shape
    K = w.shape[1]
    if w.shape[0] != C or hist.shape != (B, K - 1, C):
        raise ValueError("short_conv: inconsistent shape")
    y = np.zeros((B, T, C))
    h_out = np.zeros((B, K - 1, C)) if write_history else None
    L = None if accept_len is None else np.ascontiguousarray(accept_len, dtype=np.int32)
    bad = _load().oracle_short_conv(B, T, C, K, _p(x), _p(w), _p(hist), _pi(L), _p(y), _p(h_out))
    return y, h_out, int(bad)


def conv_channels(q, k, v):
    """Pack q, k [B, T, H_k, d_k] and v [B, T, H_v, d_v] into the channel order of the
    short convolution: [q heads | k heads | v heads], i.e. [B, T, 2 H_k d_k + H_v d_v]."""
    B, T = v.shape[0], v.shape[1]
    return np.concatenate([_f64(q).reshape(B, T, -1), _f64(k).reshape(B, T, -1),
                           _f64(v).reshape(B, T, -1)], axis=2)


def short_conv(q, k, v, w, hist, accept_len=None, write_history=True):
    """The short convolution applied to the mixer's q, k, v (channel order q | k | v).

    q, k: [B, T, H_k, d_k]; v: [B, T, H_v, d_v]; w: [C, K]; hist: [B, K-1, C].
    Returns (q', k', v', new history, number of out-of-range counts).
    """
    y, h_out, bad = short_conv_channels(conv_channels(q, k, v), w, hist, accept_len, write_history)
    nq, nk = int(np.prod(q.shape[2:])), int(np.prod(k.shape[2:]))
    return (y[:, :, :nq].reshape(q.shape), y[:, :, nq:nq + nk].reshape(k.shape),
            y[:, :, nq + nk:].reshape(v.shape), h_out, bad)


def gated_rmsnorm(o, z, w, eps=1e-6):
    """Gated RMS normalisation over the last axis (oracle_gated_rmsnorm):
    y = o / sqrt(mean(o^2) + eps) * w * silu(z). o, z: [..., d]; w: [d]."""
    o, z, w = _f64(o), _f64(z), _f64(w)
    d = o.shape[-1]
    if z.shape != o.shape or w.shape != (d,):
        raise ValueError("gated_rmsnorm: inconsistent shape")
    y = np.empty_like(o)
    _load().oracle_gated_rmsnorm(o.size // d if d else 0, d, _p(o), _p(z), _p(w), float(eps), _p(y))
    return y


def accept(target, tokens, draft=None, u=None, tau=1.0, sampled=False):
    """Acceptance of verify blocks (oracle_accept).

    target: [B, T, V] logits; tokens: [B, T] int (row 0 the anchor); draft: [B, T-1, V] logits
    and u: [B, T] uniforms in sampled mode. Returns (accept_len [B], next_token [B], pd, qd):
    pd / qd [B, T-1] are p_t and q_t at each draft token (greedy: pd holds the argmax).
    """
    target = _f64(target)
    B, T, V = target.shape
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    d = None if draft is None else _f64(draft)
    uu = None if u is None else _f64(u)
    L = np.zeros(B, dtype=np.int32)
    nt = np.zeros(B, dtype=np.int32)
    pd = np.zeros((B, max(T - 1, 1)))
    qd = np.zeros((B, max(T - 1, 1)))
    rc = _load().oracle_accept(B, T, V, _p(target), _p(d), _pi(tok), _p(uu), float(tau), int(bool(sampled)),
                               _pi(L), _pi(nt), _p(pd), _p(qd))
    if rc != 0:
        raise ValueError("oracle_accept: bad arguments")
    return L, nt, pd[:, :T - 1], qd[:, :T - 1]
