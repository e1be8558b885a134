"""Seeded synthetic inputs for the Gated DeltaNet verify / decode / prefill mixer.

This module draws random numbers and rounds them to their storage type; it holds
none of the mixer's arithmetic. Both the CUDA path's tests / benchmark and the
CPU oracle take their inputs from here.

Workloads (the shapes of the source pages' target: a 64-layer hybrid whose 48
Gated DeltaNet layers each carry a 32-bit recurrent state, verified in blocks
of 7 drafted tokens plus 1 anchor, with a 32K context -- "Qwen 3.8 27B mac m5:
200 tok/s, audited", sections on fusing layer mixers and on DSpark; and
"Lithos-metal: Qwen3.8-27B on 40-core M5 Max", quick start, 32K context):

  tiny_verify          B=1,   1 layer,  H_k=H_v=2,   d=16,  T=8, fp32 inputs
  single_seq_verify    B=1,  48 layers, H_k=16/H_v=48, d=128, T=8, bf16 q/k/v/a/b
  batched_verify       B=64,  1 layer,  H_k=16/H_v=48, d=128, T=8, bf16
  decode               B=256, 1 layer,  H_k=16/H_v=48, d=128, T=1, bf16
  prefill              B=1,   1 layer,  H_k=16/H_v=48, d=128, T=32768, chunk 64, bf16

Distributions: q, k, v, a, b ~ N(0, 1); A_log ~ U(ln 1, ln 16); dt_bias = 0;
initial state ~ N(0, sigma) with sigma 0.1 (tiny), 0.05 (model-scale), zero for
prefill; accept_len ~ U{1..8} (tiny) or min(Geometric(0.25), 8) with support
{1, 2, ...} (model-scale verify). Draw order per (workload, layer) stream:
S0, q, k, v, a, b, A_log, accept_len. bf16 tensors are rounded once, here,
round-to-nearest-even, by torch's float32 -> bfloat16 conversion.
"""
from dataclasses import dataclass, replace
from typing import Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H_k: int
    H_v: int
    d_k: int
    d_v: int
    layers: int = 1
    in_dtype: str = "bf16"          # storage type of q, k, v, a, b
    state_std: float = 0.05         # 0 -> zero initial state
    accept: str = "geometric"       # "uniform", "geometric", "all" (commit T), "none"
    chunk: int = 0                  # prefill chunk length (0: not a prefill workload)
    seed: int = 1000


WORKLOADS = {
    "tiny_verify": Workload("tiny_verify", B=1, T=8, H_k=2, H_v=2, d_k=16, d_v=16,
                            in_dtype="f32", state_std=0.1, accept="uniform", seed=1000),
    "single_seq_verify": Workload("single_seq_verify", B=1, T=8, H_k=16, H_v=48, d_k=128,
                                  d_v=128, layers=48, seed=1001),
    "batched_verify": Workload("batched_verify", B=64, T=8, H_k=16, H_v=48, d_k=128, d_v=128,
                               seed=1002),
    "decode": Workload("decode", B=256, T=1, H_k=16, H_v=48, d_k=128, d_v=128, accept="all",
                       seed=1003),
    "prefill": Workload("prefill", B=1, T=32768, H_k=16, H_v=48, d_k=128, d_v=128,
                        state_std=0.0, accept="none", chunk=64, seed=1004),
}

# Index of each workload in the list of configurations it was specified as.
CONFIG_ORDER = ["tiny_verify", "single_seq_verify", "batched_verify", "decode", "prefill"]


def workload(name_or_index, **overrides) -> Workload:
    """A named (or indexed) workload, with optional field overrides (B, T, seed, ...)."""
    name = CONFIG_ORDER[name_or_index] if isinstance(name_or_index, int) else name_or_index
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def _store(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def make_inputs(w: Workload, layer: int = 0, gates: str = "config",
                accept_len: Optional[np.ndarray] = None) -> dict:
    """Draw one layer's inputs for workload ``w`` (CPU torch tensors).

    gates: "config" (a, b ~ N(0, 1)) or "gentle" (a ~ N(-6, 1): decays near 0.99, so the
    initial state stays visible in the outputs).
    Returns q, k [B,T,H_k,d_k]; v [B,T,H_v,d_v]; a, b [B,T,H_v] (in_dtype); A_log, dt_bias
    [H_v] fp32; S0 [B,H_v,d_v,d_k] fp32; accept_len [B] int32 or None.
    """
    rng = np.random.default_rng([w.seed, layer])
    B, T, Hk, Hv, dk, dv = w.B, w.T, w.H_k, w.H_v, w.d_k, w.d_v
    f32 = np.float32
    if w.state_std > 0:
        S0 = rng.standard_normal((B, Hv, dv, dk), dtype=f32) * f32(w.state_std)
    else:
        S0 = np.zeros((B, Hv, dv, dk), dtype=f32)
    q = rng.standard_normal((B, T, Hk, dk), dtype=f32)
    k = rng.standard_normal((B, T, Hk, dk), dtype=f32)
    v = rng.standard_normal((B, T, Hv, dv), dtype=f32)
    a = rng.standard_normal((B, T, Hv), dtype=f32)
    if gates == "gentle":
        a = a - f32(6.0)
    elif gates != "config":
        raise ValueError(gates)
    b = rng.standard_normal((B, T, Hv), dtype=f32)
    A_log = rng.uniform(np.log(1.0), np.log(16.0), size=Hv).astype(f32)
    dt_bias = np.zeros(Hv, dtype=f32)
    if accept_len is not None:
        L = np.ascontiguousarray(accept_len, dtype=np.int32)
    elif w.accept == "uniform":
        L = rng.integers(1, T + 1, size=B).astype(np.int32)
    elif w.accept == "geometric":
        L = np.minimum(rng.geometric(0.25, size=B), T).astype(np.int32)
    elif w.accept == "all":
        L = np.full(B, T, dtype=np.int32)
    elif w.accept == "none":
        L = None
    else:
        raise ValueError(w.accept)
    return {
        "q": _store(q, w.in_dtype), "k": _store(k, w.in_dtype), "v": _store(v, w.in_dtype),
        "a": _store(a, w.in_dtype), "b": _store(b, w.in_dtype),
        "A_log": torch.from_numpy(A_log), "dt_bias": torch.from_numpy(dt_bias),
        "S0": torch.from_numpy(S0),
        "accept_len": None if L is None else torch.from_numpy(L),
    }


def make_conv_inputs(w: Workload, K: int = 4, layer: int = 0) -> dict:
    """Synthetic short-convolution parameters for workload ``w`` (CPU torch tensors):
    conv_w [C, K] fp32 ~ U(-1/sqrt(K), 1/sqrt(K)) (a depthwise filter's default init) and
    hist [B, K-1, C] ~ N(0, 1) in the workload's input dtype, C = 2 H_k d_k + H_v d_v
    (channels q | k | v). Its own stream, (seed, layer, 7), so the mixer inputs are unchanged."""
    rng = np.random.default_rng([w.seed, layer, 7])
    C = 2 * w.H_k * w.d_k + w.H_v * w.d_v
    bound = 1.0 / np.sqrt(K)
    conv_w = rng.uniform(-bound, bound, size=(C, K)).astype(np.float32)
    hist = rng.standard_normal((w.B, K - 1, C), dtype=np.float32)
    return {"conv_w": torch.from_numpy(conv_w), "hist": _store(hist, w.in_dtype)}


def make_conv_block(w: Workload, K: int = 4, layer: int = 0) -> dict:
    """One layer's inputs of the short convolution alone (no recurrent state): q, k, v
    ~ N(0, 1) before the convolution (the workload's layouts and input dtype), accept_len as
    the workload draws it, and conv_w, hist as :func:`make_conv_inputs`. Its own stream,
    (seed, layer, 8)."""
    rng = np.random.default_rng([w.seed, layer, 8])
    B, T, Hk, Hv, dk, dv = w.B, w.T, w.H_k, w.H_v, w.d_k, w.d_v
    f32 = np.float32
    q = rng.standard_normal((B, T, Hk, dk), dtype=f32)
    k = rng.standard_normal((B, T, Hk, dk), dtype=f32)
    v = rng.standard_normal((B, T, Hv, dv), dtype=f32)
    L = np.minimum(rng.geometric(0.25, size=B), T).astype(np.int32)
    out = {"q": _store(q, w.in_dtype), "k": _store(k, w.in_dtype), "v": _store(v, w.in_dtype),
           "accept_len": torch.from_numpy(L)}
    out.update(make_conv_inputs(w, K=K, layer=layer))
    return out


def make_norm_inputs(w: Workload, layer: int = 0) -> dict:
    """Synthetic inputs of the gated output normalisation: the gate z ~ N(0, 1) with v's shape
    [B, T, H_v, d_v] in the input dtype, and the weight norm_w ~ U(0.5, 1.5) [d_v] fp32. Its own
    stream, (seed, layer, 9)."""
    rng = np.random.default_rng([w.seed, layer, 9])
    z = rng.standard_normal((w.B, w.T, w.H_v, w.d_v), dtype=np.float32)
    nw = rng.uniform(0.5, 1.5, size=w.d_v).astype(np.float32)
    return {"norm_z": _store(z, w.in_dtype), "norm_w": torch.from_numpy(nw)}


def make_accept_inputs(w: Workload, V: int = 151936, layer: int = 0, plant: float = 0.8,
                       dtype: Optional[str] = None) -> dict:
    """Synthetic acceptance inputs for blocks of workload ``w`` (B sequences of T rows) over a
    vocabulary of V: target logits ~ N(0, 1) [B, T, V]; draft logits = the target's first T-1
    rows + N(0, 0.5) noise; tokens [B, T] uniform over V (row 0 the anchor); uniforms [B, T] ~
    U[0, 1). At a fraction `plant` of the draft positions, both models get +8 on the drafted
    token's logit (so that acceptance runs look like a real drafter's). Logits are stored in
    `dtype` (default the workload's input dtype). Its own stream, (seed, layer, 10)."""
    rng = np.random.default_rng([w.seed, layer, 10])
    B, T = w.B, w.T
    f32 = np.float32
    target = rng.standard_normal((B, T, V), dtype=f32)
    draft = target[:, :T - 1] + f32(0.5) * rng.standard_normal((B, T - 1, V), dtype=f32)
    tokens = rng.integers(0, V, size=(B, T)).astype(np.int32)
    planted = rng.random((B, T - 1)) < plant
    bi, ti = np.nonzero(planted)
    target[bi, ti, tokens[bi, ti + 1]] += f32(8.0)
    draft[bi, ti, tokens[bi, ti + 1]] += f32(8.0)
    u = rng.random((B, T)).astype(f32)
    dt = dtype or w.in_dtype
    return {"target": _store(target, dt), "draft": _store(draft, dt), "tokens": torch.from_numpy(tokens),
            "uniforms": torch.from_numpy(u)}


def as_f64(inputs: dict) -> dict:
    """The same inputs as float64 NumPy arrays (exact: every stored value is representable)."""
    out = {}
    for key, val in inputs.items():
        if val is None:
            out[key] = None
        elif key == "accept_len":
            out[key] = val.numpy().astype(np.int32)
        else:
            out[key] = val.to(torch.float64).numpy()
    return out

