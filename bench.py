"""Benchmark of the Gated DeltaNet verify mixer on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload all|batched_verify|decode|single_seq_verify|prefill|...]

A step is one pass of the mixer over one batch of synthetic input, through the C ABI:
  batched_verify     (default) 64 sequences x 48 value heads, a 7 + 1 verify block, the
                     committed state written at each sequence's device-side accept count
  decode             256 sequences, one token each, state updated in place
  single_seq_verify  one sequence through 48 distinct layers, replayed as a CUDA graph
  prefill            one 32768-token prompt, chunk 64
The default (`all`) prints batched_verify as the headline line and nests one record per other
workload under "configs" (decode, prefill, single_seq_verify, then commit_next_verify,
verify_gated, short_conv, accept, accept_greedy), each with its own step time, roofline,
clocks, e2e leg and CPU-oracle sample; `--workload NAME` prints that workload alone.
Under torchrun each rank runs its own batch (weak scaling, no data-path collective); the
step time is the max over ranks. `--impl reference` times the fp64 CPU oracle instead, on
a bounded sample of the same workload, on rank 0 only.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_deltanet_mixer_verify_b200.dist import max_over_ranks, rank_seed, weak_scaling_throughput  # noqa: E402
from gated_deltanet_mixer_verify_b200.inputs import make_inputs, workload  # noqa: E402

METRIC = "GDN verify/decode HBM GB/s (frac of B200 peak), token·heads/s; prefill tok/s"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
NOMINAL_TF32_OVER_BF16 = 1.1 / 2.25     # dense tensor-core peaks, tf32 vs bf16
# Sources of each workload's dominant kernel (with the headers it includes); a committed ncu
# traffic figure is only reported while these are unchanged.
_CSRC = "gated_deltanet_mixer_verify_b200/csrc/"
_HEADERS = [_CSRC + f for f in ("gdn_tc.cuh", "gdn_device.cuh", "gdn_internal.cuh")]
KERNEL_SOURCES = {
    "batched_verify": [_CSRC + "gdn_verify.cu", _CSRC + "gdn_verify_pipe.cu"] + _HEADERS,
    "commit_next_verify": [_CSRC + "gdn_verify.cu", _CSRC + "gdn_verify_tc.cu"] + _HEADERS,
    "verify_gated": [_CSRC + "gdn_verify.cu", _CSRC + "gdn_verify_tc.cu"] + _HEADERS,
    "decode": [_CSRC + "gdn_verify.cu", _CSRC + "gdn_verify_head.cu"] + _HEADERS,
    "single_seq_verify": [_CSRC + "gdn_verify.cu", _CSRC + "gdn_verify_rec.cu"] + _HEADERS,
    "prefill": [_CSRC + "gdn_prefill.cu", _CSRC + "gdn_prefill.cuh"] + _HEADERS,
    "short_conv": [_CSRC + "gdn_conv.cu"] + _HEADERS,
    "accept": [_CSRC + "gdn_accept.cu"] + _HEADERS,
    "accept_greedy": [_CSRC + "gdn_accept.cu"] + _HEADERS,
}
ACCEPT_V = 151936   # vocabulary of the acceptance workloads (the pages give none: the Qwen tokenizer's)
CONV_K, CONV_LAYERS = 4, 48   # short convolution: filter taps; one convolution per GDN layer


# ----------------------------------------------------------------------------- helpers

FALLBACK_BF16_TFLOPS = 1590.0


def measured_peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, source) from MEASURED_PEAKS.json, else the fallbacks."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def kernel_source_hash(workload_name: str) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[workload_name]:
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(workload_name: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary, or None
    when there is none for this workload or the kernel source changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path)).get(workload_name)
    if not d or d.get("kernel_source_sha") != kernel_source_hash(workload_name):
        return None
    return d.get("dram_bytes_per_launch")


def algorithmic_bytes(w, n_state_writes=None):
    """Bytes one verify / decode call must move: state read + committed state written, the
    per-token inputs, the gate parameters, the fp32 outputs and the accept counts."""
    el = 2 if w.in_dtype == "bf16" else 4
    B, T, Hk, Hv, dk, dv = w.B, w.T, w.H_k, w.H_v, w.d_k, w.d_v
    state = B * Hv * dv * dk * 4
    writes = B if n_state_writes is None else n_state_writes
    return (state + writes * Hv * dv * dk * 4 + 2 * B * T * Hk * dk * el + B * T * Hv * dv * el
            + 2 * B * T * Hv * el + 2 * Hv * 4 + B * T * Hv * dv * 4 + B * 4)


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None

    def _sample(self):
        p = self.nvml
        self.samples.append(p.nvmlDeviceGetClockInfo(self.h, p.NVML_CLOCK_SM))
        mask = p.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        for bit, name in self.REASONS.items():
            if mask & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.nvml:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- workloads

def stash_floats_per_head(T, dk, dv):
    """Floats of one (sequence, value head) stash: khat [T][d_k], G [T] and u [T][d_v], the
    last two padded to a multiple of 4."""
    pad = lambda n: (n + 3) // 4 * 4
    return T * dk + pad(T) + pad(T * dv)


def commit_next_bytes(w):
    """Bytes one commit-on-next-verify call must move: the verify call's (the state written
    back for every sequence) plus the previous block's stash read and this block's written."""
    stash = w.B * w.H_v * stash_floats_per_head(w.T, w.d_k, w.d_v) * 4
    return algorithmic_bytes(w, n_state_writes=w.B) + 2 * stash


def conv_bytes(w, K=CONV_K):
    """Bytes one short-convolution launch must move: q, k, v read and written once, the
    history read and rewound, the taps and the accept counts."""
    el = 2 if w.in_dtype == "bf16" else 4
    C = 2 * w.H_k * w.d_k + w.H_v * w.d_v
    return 2 * w.B * w.T * C * el + 2 * w.B * (K - 1) * C * el + C * K * 4 + w.B * 4


def gated_bytes(w):
    """Bytes of a verify call with the gated output normalisation: the verify call's, plus the
    gate z (v's size) and the d_v weights."""
    el = 2 if w.in_dtype == "bf16" else 4
    return algorithmic_bytes(w) + w.B * w.T * w.H_v * w.d_v * el + w.d_v * 4


def accept_bytes(w, sampled, V=ACCEPT_V):
    """Bytes one acceptance call must move: every logit read once (target rows, and the draft
    rows in sampled mode), the tokens, the uniforms and the two outputs."""
    el = 2 if w.in_dtype == "bf16" else 4
    n = w.B * w.T * V * el + (w.B * (w.T - 1) * V * el if sampled else 0)
    return n + w.B * w.T * 4 + (w.B * w.T * 4 if sampled else 0) + 2 * w.B * 4


def workload_config(name):
    """The JSON `config` of a workload (what it is, with its sizes)."""
    if name in ("accept", "accept_greedy"):
        w = workload("batched_verify")
        sampled = name == "accept"
        return {"workload": name, "B": w.B, "T": w.T, "V": ACCEPT_V, "logits": "bf16",
                "mode": "exact speculative sampling, temperature 1" if sampled else "greedy",
                "inputs": "target logits N(0,1) [B,T,V]" + (", draft logits target + N(0,0.5) [B,T-1,V], uniforms"
                                                             if sampled else "") +
                          "; 80% of drafted tokens planted with +8 in both models",
                "l2": "inputs larger than L2 (%.0f MB moved per step, L2 126 MB)" % (accept_bytes(w, sampled) / 1e6)}
    if name == "verify_gated":
        c = workload_config("batched_verify")
        w = workload("batched_verify")
        c.update(workload=name, norm="o / sqrt(mean(o^2) + 1e-6) * w * silu(z) per (token, value head), "
                 "z bf16 like v, w fp32 [d_v]; fused into the verify kernel's outputs",
                 l2="inputs larger than L2 (%.0f MB moved per step, L2 126 MB)" % (gated_bytes(w) / 1e6))
        return c
    if name == "short_conv":
        c = workload_config("batched_verify")
        w = workload("batched_verify")
        c.update(workload=name, conv_k=CONV_K, layers=CONV_LAYERS,
                 channels="q | k | v: %d" % (2 * w.H_k * w.d_k + w.H_v * w.d_v),
                 accept_len="min(Geometric(0.25), 8) per sequence, device int32",
                 state="short history [B, K-1, C] bf16 per layer, rewound in place",
                 launch="%d launches (one per layer, distinct buffers) captured in one CUDA graph" % CONV_LAYERS,
                 l2="inputs larger than L2 (%.0f MB moved per step, L2 126 MB)" % (conv_bytes(w) * CONV_LAYERS / 1e6))
        return c
    if name == "commit_next_verify":
        c = workload_config("batched_verify")
        w = workload("batched_verify")
        c.update(workload=name, accept_len="the previous block's: min(Geometric(0.25), 8) per "
                 "sequence, device int32",
                 state="fp32 [B,H_v,d_v,d_k]: the previous block committed in place, this "
                 "block's stash written (two-phase)",
                 l2="inputs larger than L2 (%.0f MB moved per step, L2 126 MB)" % (commit_next_bytes(w) / 1e6))
        return c
    w = workload(name)
    c = {"workload": w.name, "B": w.B, "T": w.T, "H_k": w.H_k, "H_v": w.H_v, "d_k": w.d_k,
         "d_v": w.d_v, "layers": w.layers, "in_dtype": w.in_dtype}
    if name == "batched_verify":
        c["accept_len"] = "min(Geometric(0.25), 8) per sequence, device int32"
        c["state"] = "fp32 [B,H_v,d_v,d_k], committed in place"
    elif name == "decode":
        c["state"] = "fp32 [B,H_v,d_v,d_k], updated in place"
    elif name == "single_seq_verify":
        c["accept_len"] = "one min(Geometric(0.25), 8) per round, device int32"
        c["launch"] = "48 launches captured in one CUDA graph, each a programmatic dependent of the one before"
    else:
        c["chunk"] = w.chunk
        c["state_in"] = "zero"
    if name == "prefill":
        c["l2"] = "inputs larger than L2"
    else:
        n = algorithmic_bytes(w) * w.layers
        c["l2"] = "inputs larger than L2 (%.0f MB moved per step, L2 126 MB)" % (n / 1e6)
    return c


class Verify:
    """batched_verify / decode: one C-ABI call per step over the whole batch."""

    def __init__(self, name, rank, dev):
        from gated_deltanet_mixer_verify_b200 import gdn
        self.gdn = gdn
        self.w = workload(name, seed=rank_seed(workload(name).seed, rank))
        self.decode = name == "decode"
        x = make_inputs(self.w)
        self.host = x
        self.x = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
        self.state = self.x["S0"].clone()
        self.o = torch.empty(self.x["v"].shape, dtype=torch.float32, device=dev)
        self.launches_per_step = 1
        self.bytes = algorithmic_bytes(self.w)
        self.units = self.w.B * self.w.T * self.w.H_v          # token x heads per step

    def step(self, x=None, o=None):
        x = x or self.x
        o = self.o if o is None else o
        if self.decode:
            self.gdn.decode_step(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"],
                                 x["dt_bias"], self.state, o)
        else:
            self.gdn.verify_step(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"],
                                 x["dt_bias"], self.state, self.state, x["accept_len"], o)

    def config(self):
        return workload_config(self.w.name)

    def per_step_inputs(self):
        return ["q", "k", "v", "a", "b"] + ([] if self.decode else ["accept_len"])


class VerifyGated(Verify):
    """verify_gated: batched verify whose outputs carry the gated RMS normalisation (one call,
    the normalisation applied by the verify kernel to its outputs)."""

    def __init__(self, name, rank, dev):
        super().__init__("batched_verify", rank, dev)
        from gated_deltanet_mixer_verify_b200.inputs import make_norm_inputs
        n = make_norm_inputs(self.w)
        self.host.update(n)
        self.x.update({k: v.to(dev) for k, v in n.items()})
        self.bytes = gated_bytes(self.w)

    def step(self, x=None, o=None):
        x = x or self.x
        o = self.o if o is None else o
        self.gdn.verify_step_gated(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"], self.state,
                                   self.state, x["accept_len"], x["norm_z"], x["norm_w"], 1e-6, o=o)

    def per_step_inputs(self):
        return super().per_step_inputs() + ["norm_z"]

    def config(self):
        return workload_config("verify_gated")


class CommitNext(Verify):
    """commit_next_verify: the serving loop's form of a verify step. Each call applies the
    previous block's stash at its accept counts (known by now) and verifies the next block on
    the committed state, writing that block's stash for the next call; two stash buffers
    alternate."""

    def __init__(self, name, rank, dev):
        super().__init__("batched_verify", rank, dev)
        w = self.w
        n = w.B * w.H_v * stash_floats_per_head(w.T, w.d_k, w.d_v)
        self.stash = [torch.zeros(n, dtype=torch.float32, device=dev) for _ in range(2)]
        x = self.x
        self.gdn.verify_step(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                             self.state, None, None, self.o, stash=self.stash[0])
        self.k = 0
        self.bytes = commit_next_bytes(w)

    def step(self, x=None, o=None):
        x = x or self.x
        o = self.o if o is None else o
        prev, cur = self.stash[self.k & 1], self.stash[(self.k + 1) & 1]
        self.gdn.commit_and_verify(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                                   self.state, prev, x["accept_len"], self.w.T, o=o, stash=cur)
        self.k += 1

    def config(self):
        return workload_config("commit_next_verify")


class ShortConv:
    """short_conv: the causal short convolution of one verify block (B = 64, T = 8) for each of
    48 layers, each with its own inputs, taps and history, captured once as a CUDA graph; a
    step replays the graph."""

    def __init__(self, name, rank, dev):
        from gated_deltanet_mixer_verify_b200 import gdn
        from gated_deltanet_mixer_verify_b200.inputs import make_conv_block
        self.gdn = gdn
        self.w = workload("batched_verify", seed=rank_seed(workload("batched_verify").seed, rank))
        self.layers = []
        for l in range(CONV_LAYERS):
            x = make_conv_block(self.w, K=CONV_K, layer=l)
            if l == 0:
                self.host = x
            xd = {k: v.to(dev) for k, v in x.items()}
            xd.update(qo=torch.empty_like(xd["q"]), ko=torch.empty_like(xd["k"]), vo=torch.empty_like(xd["v"]))
            self.layers.append(xd)
        self.launches_per_step = CONV_LAYERS
        self.bytes = conv_bytes(self.w) * CONV_LAYERS
        self.units = self.w.B * self.w.T * self.w.H_v * CONV_LAYERS
        self.graph = None
        self.stream = torch.cuda.Stream(dev)

    def conv(self, x):
        self.gdn.short_conv(x["q"], x["k"], x["v"], x["conv_w"], x["hist"], x["hist"], x["accept_len"],
                            q_out=x["qo"], k_out=x["ko"], v_out=x["vo"], stream=self.stream)

    def step(self):
        if self.graph is None:
            with torch.cuda.stream(self.stream):
                for x in self.layers:
                    self.conv(x)                                  # warm the launch path
            torch.cuda.current_stream().wait_stream(self.stream)
            torch.cuda.synchronize()
            self.graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.graph, stream=self.stream):
                for x in self.layers:
                    self.conv(x)
        self.graph.replay()

    def e2e(self, steps, barrier, world, dev):
        """Through the public call with host buffers: per step, one layer's q, k, v and accept
        counts copied in from pinned memory, the convolution, its q', k', v' copied out."""
        names = ["q", "k", "v", "accept_len"]
        host = {k: self.host[k].pin_memory() for k in names}
        x = dict(self.layers[0])
        x.update({k: torch.empty_like(self.layers[0][k]) for k in names})
        outs = [torch.empty(x[k].shape, dtype=x[k].dtype).pin_memory() for k in ("qo", "ko", "vo")]
        stream = torch.cuda.current_stream(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(steps):
            for k in names:
                x[k].copy_(host[k], non_blocking=True)
            self.gdn.short_conv(x["q"], x["k"], x["v"], x["conv_w"], x["hist"], x["hist"], x["accept_len"],
                                q_out=x["qo"], k_out=x["ko"], v_out=x["vo"])
            for o, k in zip(outs, ("qo", "ko", "vo")):
                o.copy_(x[k], non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e_s = max_over_ranks(e0.elapsed_time(e1)) / steps / 1e3
        h2d = sum(host[k].numel() * host[k].element_size() for k in names)
        d2h = sum(o.numel() * o.element_size() for o in outs)
        return {"value": weak_scaling_throughput(conv_bytes(self.w), world, e_s) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    def config(self):
        return workload_config("short_conv")


class Accept:
    """accept / accept_greedy: device-side acceptance of a batch of verify blocks (B = 64, T = 8,
    V = 151,936 bf16 logits): one C-ABI call per step (two kernels)."""

    def __init__(self, name, rank, dev):
        from gated_deltanet_mixer_verify_b200 import gdn
        from gated_deltanet_mixer_verify_b200.inputs import make_accept_inputs
        self.gdn = gdn
        self.name = name
        self.sampled = name == "accept"
        self.w = workload("batched_verify", seed=rank_seed(workload("batched_verify").seed, rank))
        self.host = make_accept_inputs(self.w, V=ACCEPT_V)
        self.x = {k: v.to(dev) for k, v in self.host.items()}
        B, T = self.w.B, self.w.T
        self.ws = torch.empty(gdn.accept_workspace_bytes(B, T, ACCEPT_V, self.sampled), dtype=torch.uint8, device=dev)
        self.L = torch.empty(B, dtype=torch.int32, device=dev)
        self.o = torch.empty(B, dtype=torch.int32, device=dev)   # the next tokens
        self.launches_per_step = 2 if self.sampled else 1
        self.calls_per_step = 1
        self.bytes = accept_bytes(self.w, self.sampled)
        self.units = B * T

    def step(self, x=None):
        x = x or self.x
        self.gdn.accept(x["target"], x["tokens"], x["draft"] if self.sampled else None,
                        x["uniforms"] if self.sampled else None, workspace=self.ws, accept_len=self.L,
                        next_token=self.o)

    def per_step_inputs(self):
        return ["target", "tokens"] + (["draft", "uniforms"] if self.sampled else [])

    def config(self):
        return workload_config(self.name)


class SingleSeq:
    """single_seq_verify: one sequence through 48 distinct layers, one launch per layer,
    captured once as a CUDA graph; a step replays the graph. Each input kind of all layers
    lives in one device buffer (layer l reads slice l), and the round's one accept count in
    one int32, so that a round's inputs arrive in one copy per kind."""

    KINDS = ("q", "k", "v", "a", "b")

    def __init__(self, name, rank, dev):
        from gated_deltanet_mixer_verify_b200 import gdn
        self.gdn = gdn
        self.w = workload(name, seed=rank_seed(workload(name).seed, rank))
        L0 = make_inputs(self.w, layer=0)["accept_len"]
        xs = [make_inputs(self.w, layer=l, accept_len=L0.numpy()) for l in range(self.w.layers)]
        self.host = {k: torch.stack([x[k] for x in xs]) for k in self.KINDS}
        self.host["accept_len"] = L0.clone()
        self.dev = {k: v.to(dev) for k, v in self.host.items()}
        self.o_all = torch.empty((self.w.layers,) + tuple(xs[0]["v"].shape), dtype=torch.float32, device=dev)
        self.layers = []
        for l, x in enumerate(xs):
            xd = {k: self.dev[k][l] for k in self.KINDS}
            xd.update(A_log=x["A_log"].to(dev), dt_bias=x["dt_bias"].to(dev), state=x["S0"].to(dev),
                      accept_len=self.dev["accept_len"], o=self.o_all[l])
            self.layers.append(xd)
        self.launches_per_step = self.w.layers
        self.bytes = algorithmic_bytes(self.w) * self.w.layers
        self.units = self.w.B * self.w.T * self.w.H_v * self.w.layers
        self.graph = None
        self.stream = torch.cuda.Stream(dev)

    def _eager(self):
        # Programmatic dependent launch: each layer's kernel stages its own state while the
        # previous layer's runs (a layer's state was last written by its own previous call).
        for x in self.layers:
            self.gdn.verify_step(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"],
                                 x["dt_bias"], x["state"], x["state"], x["accept_len"], x["o"], pdl=True)

    def step(self):
        if self.graph is None:
            with torch.cuda.stream(self.stream):
                self._eager()                                     # warm the launch path
            torch.cuda.current_stream().wait_stream(self.stream)
            torch.cuda.synchronize()
            self.graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.graph, stream=self.stream):
                self._eager()
        self.graph.replay()

    def e2e(self, steps, barrier, world, dev):
        """Through the public calls with host buffers: per round, every layer's q, k, v, a, b and
        the round's accept count copied in from pinned memory (one copy per kind), the 48
        launches (the graph), every layer's o copied out (one copy)."""
        self.step()
        host = {k: v.pin_memory() for k, v in self.host.items()}
        o_host = torch.empty(self.o_all.shape, dtype=self.o_all.dtype).pin_memory()
        s = self.stream
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(s):
            e0.record(s)
            for _ in range(steps):
                for k, h in host.items():
                    self.dev[k].copy_(h, non_blocking=True)
                self.graph.replay()
                o_host.copy_(self.o_all, non_blocking=True)
            e1.record(s)
        torch.cuda.synchronize(dev)
        barrier()
        e_s = max_over_ranks(e0.elapsed_time(e1)) / steps / 1e3
        h2d = sum(h.numel() * h.element_size() for h in host.values())
        return {"value": weak_scaling_throughput(self.bytes, world, e_s) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": o_host.numel() * o_host.element_size()}

    def config(self):
        return workload_config(self.w.name)


class Prefill:
    tokens = 0   # prompt length override (0: the workload's)
    dtype = "tf32"   # tensor-core products in tf32 (one or two passes), solves in fp32

    def __init__(self, name, rank, dev):
        from gated_deltanet_mixer_verify_b200 import gdn
        self.gdn = gdn
        self.w = workload(name, seed=rank_seed(workload(name).seed, rank))
        if Prefill.tokens:
            self.w = workload(name, seed=self.w.seed, T=Prefill.tokens)
        self.host = make_inputs(self.w)
        self.x = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in self.host.items()}
        w = self.w
        self.o = torch.empty(self.x["v"].shape, dtype=torch.float32, device=dev)
        self.state = torch.empty((w.B, w.H_v, w.d_v, w.d_k), dtype=torch.float32, device=dev)
        nb = gdn.prefill_workspace_bytes(w.B, w.T, w.H_k, w.H_v, w.d_k, w.d_v, w.chunk)
        self.ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=dev)
        # the prompt runs in pieces, each a prepare launch and a scan launch
        self.launches_per_step = 2 * gdn.chunk_prefill_pieces(self.w.T, self.w.chunk)
        self.units = w.B * w.T
        C, dk, dv = w.chunk, w.d_k, w.d_v
        n_units = w.B * w.H_v * ((w.T + C - 1) // C)
        # Algorithmic work per (sequence, value head, chunk). Scan (tensor cores, counted once
        # however many tf32 passes carry it): [P | R] = S [Khat; Qhat]^T, the state update
        # X Keff and the outputs X Mo^T. Prepare (CUDA cores): the 192 triangular row solves
        # giving Mo and Keff^T, 63 * 64 / 2 fused multiply-adds each.
        self.phase_names = ["prepare", "scan"]
        self.phase_work = [n_units * 192 * (63 * 64 // 2) * 2,
                           n_units * (2 * dv * dk * 2 * C + 2 * dv * C * dk + 2 * dv * C * C)]
        self.phase_kernel = ["gdn_prefill_prep_kernel", "gdn_prefill_scan_kernel"]

    def phases(self, x=None):
        x = self.x if x is None else x
        g, w = self.gdn, self.w
        return [lambda: g.chunk_prefill_prepare(x["q"], x["k"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                                                self.ws, chunk=w.chunk),
                lambda: g.chunk_prefill_scan(x["v"], self.ws, w.H_k, None, self.state, self.o, chunk=w.chunk)]

    def step(self, x=None):
        # the public one-call prefill: pieces, the scan of one beside the prepare of the next
        x = self.x if x is None else x
        w = self.w
        self.gdn.chunk_prefill(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"], None,
                               self.state, self.o, chunk=w.chunk, workspace=self.ws)

    def per_step_inputs(self):
        return ["q", "k", "v", "a", "b"]

    def config(self):
        c = workload_config(self.w.name)
        c["T"] = self.w.T
        return c


WORKLOADS = {"batched_verify": Verify, "decode": Verify, "single_seq_verify": SingleSeq,
             "prefill": Prefill, "commit_next_verify": CommitNext, "short_conv": ShortConv,
             "verify_gated": VerifyGated, "accept": Accept, "accept_greedy": Accept}


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample(name, budget_s, rank=0):
    """Time the fp64 oracle (as it stands) on a bounded sample of the workload's units.
    Returns (seconds per unit, units timed, description, threads)."""
    from gated_deltanet_mixer_verify_b200.inputs import as_f64
    from oracle import gdn_oracle as orc
    shape = "batched_verify" if name in ("commit_next_verify", "short_conv", "verify_gated", "accept",
                                         "accept_greedy") else name
    w = workload(shape, seed=rank_seed(workload(shape).seed, rank))
    threads = orc.max_threads()
    if name in ("accept", "accept_greedy"):
        from gated_deltanet_mixer_verify_b200.inputs import make_accept_inputs
        sampled = name == "accept"
        n_seq = 4
        x = make_accept_inputs(workload(shape, B=n_seq), V=ACCEPT_V)
        f = {k: v.double().numpy() for k, v in x.items() if k != "tokens"}
        reps, t_total = 0, 0.0
        while t_total < budget_s or reps == 0:
            t0 = time.perf_counter()
            orc.accept(f["target"], x["tokens"].numpy(), f["draft"] if sampled else None,
                       f["uniforms"] if sampled else None, sampled=sampled)
            t_total += time.perf_counter() - t0
            reps += 1
            if reps >= 1000:
                break
        desc = "%d sequences x T=%d x V=%d, %s, %d repetition(s)" % (n_seq, w.T, ACCEPT_V,
                                                                     "sampled" if sampled else "greedy", reps)
        return t_total / (reps * n_seq), n_seq * reps, desc, 1
    if name == "short_conv":
        from gated_deltanet_mixer_verify_b200.inputs import make_conv_block
        n_seq = 16
        sub = workload(shape, B=n_seq)
        blk = make_conv_block(sub, K=CONV_K)
        f = {k: v.double().numpy() for k, v in blk.items() if k != "accept_len"}
        L = blk["accept_len"].numpy()
        reps, t_total = 0, 0.0
        while t_total < budget_s or reps == 0:
            t0 = time.perf_counter()
            orc.short_conv(f["q"], f["k"], f["v"], f["conv_w"], f["hist"], L)
            t_total += time.perf_counter() - t0
            reps += 1
            if reps >= 1000:
                break
        desc = "%d sequences x %d channels x T=%d, K=%d, %d repetition(s)" % (
            n_seq, 2 * w.H_k * w.d_k + w.H_v * w.d_v, w.T, CONV_K, reps)
        return t_total / (reps * n_seq), n_seq * reps, desc, 1
    if name == "prefill":
        sub = workload(name, T=2048, H_k=1, H_v=3)
        f = as_f64(make_inputs(sub))
        t0 = time.perf_counter()
        orc.prefill(f["q"], f["k"], f["v"], f["a"], f["b"], f["A_log"], f["dt_bias"], None)
        dt = time.perf_counter() - t0
        # units are tokens of all 48 heads: 3 of 48 heads timed over 2048 tokens
        per_token = dt / 2048 * (w.H_v / 3)
        return per_token, 2048, "2048 tokens x 3 of 48 value heads (fp64 recurrence)", threads
    n_seq = {"batched_verify": 8, "decode": 64, "single_seq_verify": 1, "commit_next_verify": 8,
             "verify_gated": 8}[name]
    sub = workload(shape, B=n_seq)
    f = as_f64(make_inputs(sub))
    L = f["accept_len"] if name != "decode" else None
    if name == "verify_gated":
        from gated_deltanet_mixer_verify_b200.inputs import make_norm_inputs
        nrm = {k: v.double().numpy() for k, v in make_norm_inputs(sub).items()}
    reps, t_total = 0, 0.0
    while t_total < budget_s or reps == 0:
        t0 = time.perf_counter()
        o, _, _ = orc.verify(f["q"], f["k"], f["v"], f["a"], f["b"], f["A_log"], f["dt_bias"], f["S0"], L)
        if name == "verify_gated":
            orc.gated_rmsnorm(o, nrm["norm_z"], nrm["norm_w"], 1e-6)
        t_total += time.perf_counter() - t0
        reps += 1
        if reps >= 1000:
            break
    per_seq = t_total / (reps * n_seq)
    desc = "%d sequence(s) x %d value heads x T=%d, %d repetition(s)" % (n_seq, w.H_v, w.T, reps)
    if name == "commit_next_verify":
        desc += " (one block verified and committed at its counts per sequence per step)"
    return per_seq, n_seq * reps, desc, threads


def cpu_value(name, per_unit_s):
    """The workload metric (GB/s or tok/s) the oracle reaches at per_unit_s per unit."""
    if name == "prefill":
        return 1.0 / per_unit_s, "tok/s"
    if name in ("accept", "accept_greedy"):
        per_seq_bytes = accept_bytes(workload("batched_verify", B=1), name == "accept")
    elif name == "short_conv":
        per_seq_bytes = conv_bytes(workload("batched_verify", B=1))
    elif name == "verify_gated":
        per_seq_bytes = gated_bytes(workload("batched_verify", B=1))
    elif name == "commit_next_verify":
        per_seq_bytes = commit_next_bytes(workload("batched_verify", B=1))
    else:
        per_seq_bytes = algorithmic_bytes(workload(name, B=1))
    return per_seq_bytes / per_unit_s / 1e9, "GB/s"


# ----------------------------------------------------------------------------- main

def run_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle as it stands, on the host cores, rank 0 only.
    Each step is a bounded sample of the workload (one sequence of the batch for verify,
    16 for decode, 256 tokens x 3 heads for prefill)."""
    if rank != 0:
        return
    from gated_deltanet_mixer_verify_b200.inputs import as_f64
    from oracle import gdn_oracle as orc
    name = "batched_verify" if args.workload == "all" else args.workload   # the headline's config
    if name == "prefill":
        sub = workload(name, T=256, H_k=1, H_v=3)
        f = as_f64(make_inputs(sub))
        run = lambda: orc.prefill(f["q"], f["k"], f["v"], f["a"], f["b"], f["A_log"],
                                  f["dt_bias"], None)
        units_per_step = 256 * 3 / workload(name).H_v          # prompt tokens (all heads)
        desc = "256 tokens x 3 of 48 value heads per step (fp64 recurrence)"
    elif name in ("accept", "accept_greedy"):
        from gated_deltanet_mixer_verify_b200.inputs import make_accept_inputs
        sampled = name == "accept"
        sub = workload("batched_verify", B=2)
        xa = make_accept_inputs(sub, V=ACCEPT_V)
        fa = {k: v.double().numpy() for k, v in xa.items() if k != "tokens"}
        run = lambda: orc.accept(fa["target"], xa["tokens"].numpy(), fa["draft"] if sampled else None,
                                 fa["uniforms"] if sampled else None, sampled=sampled)
        units_per_step = accept_bytes(sub, sampled) / 1e9
        desc = "2 sequences x T=8 x V=%d per step, %s" % (ACCEPT_V, "sampled" if sampled else "greedy")
    elif name == "short_conv":
        from gated_deltanet_mixer_verify_b200.inputs import make_conv_block
        sub = workload("batched_verify", B=4)
        blk = make_conv_block(sub, K=CONV_K)
        f = {k: v.double().numpy() for k, v in blk.items() if k != "accept_len"}
        L = blk["accept_len"].numpy()
        run = lambda: orc.short_conv(f["q"], f["k"], f["v"], f["conv_w"], f["hist"], L)
        units_per_step = conv_bytes(sub) / 1e9
        desc = "4 sequences x 10240 channels x T=8, K=%d per step (one layer)" % CONV_K
    else:
        n_seq = 16 if name == "decode" else 1
        shape = "batched_verify" if name in ("commit_next_verify", "verify_gated") else name
        sub = workload(shape, B=n_seq)
        f = as_f64(make_inputs(sub))
        L = None if name == "decode" else f["accept_len"]
        if name == "verify_gated":
            from gated_deltanet_mixer_verify_b200.inputs import make_norm_inputs
            nrm = {k: v.double().numpy() for k, v in make_norm_inputs(sub).items()}
            run = lambda: orc.gated_rmsnorm(orc.verify(f["q"], f["k"], f["v"], f["a"], f["b"], f["A_log"],
                                                       f["dt_bias"], f["S0"], L)[0],
                                            nrm["norm_z"], nrm["norm_w"], 1e-6)
        else:
            run = lambda: orc.verify(f["q"], f["k"], f["v"], f["a"], f["b"], f["A_log"],
                                     f["dt_bias"], f["S0"], L)
        per_step = {"commit_next_verify": commit_next_bytes, "verify_gated": gated_bytes}.get(
            name, algorithmic_bytes)(sub)
        units_per_step = per_step / 1e9                        # GB of the workload per step
        desc = "%d sequence(s) x 48 value heads x T=%d per step" % (n_seq, sub.T)
        if name == "commit_next_verify":
            desc += " (one block verified and committed at its counts)"
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    value = units_per_step * args.steps / dt
    unit = "tok/s" if name == "prefill" else "GB/s"
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference", "config": workload_config(name),
            "cpu_baseline": {"value": value, "unit": unit,
                             "cores": 1 if name in ("short_conv", "accept", "accept_greedy") else orc.max_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def measure(name, args, rank, world, dev, barrier, cpu_budget_s):
    """Time K steps of one workload after W warm-ups (every rank), and return rank 0's record
    (None on the other ranks)."""
    wl = WORKLOADS[name](name, rank, dev)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        wl.step()
    torch.cuda.synchronize(dev)

    # timed region: K steps back to back between two device events on the launching stream
    # (no event between steps: one would sit between consecutive launches and stretch them)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(torch.cuda.current_device())   # NVML set up before, not inside, the idle gap
    barrier()
    torch.cuda.synchronize(dev)
    with clk:
        start.record(stream)
        for i in range(args.steps):
            wl.step()
        end.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    local_ms = start.elapsed_time(end)
    elapsed_ms = max_over_ranks(local_ms)
    ms_per_step = elapsed_ms / args.steps

    # Per-kernel times where a step overlaps kernels on two streams (prefill: the scan of one
    # piece beside the prepare of the next), so that events cannot isolate them: a second loop
    # of K steps that runs each phase over the whole prompt, one after the other, on the
    # launching stream, with an event after each phase.
    phase_ms = None
    if hasattr(wl, "phases"):
        phases = wl.phases()
        nph = len(phases)
        pev = [[torch.cuda.Event(enable_timing=True) for _ in range(nph + 1)] for _ in range(args.steps)]
        for ph in phases:      # warm the whole-prompt launches
            ph()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            pev[i][0].record(stream)
            for j, ph in enumerate(phases):
                ph()
                pev[i][j + 1].record(stream)
        torch.cuda.synchronize(dev)
        phase_ms = [max_over_ranks(statistics.mean(e[j].elapsed_time(e[j + 1]) for e in pev))
                    for j in range(nph)]

    # end to end through the public API: pinned host inputs -> device -> mixer -> host output
    e2e = None
    if hasattr(wl, "e2e"):
        e2e = wl.e2e(args.steps, barrier, world, dev)
    elif isinstance(wl, (Verify, Prefill, Accept)):
        # Every step copies its own inputs in from pinned host memory and its result out, as a
        # serving loop does: double-buffered, on an upload and a download stream, so that step
        # i+1's inputs arrive and step i-1's result leaves while step i computes. Events order
        # each buffer's reuse (inputs after the step that read them, outputs after the copy out).
        names = wl.per_step_inputs()
        host = {k: wl.host[k].pin_memory() for k in names}
        dev_in = []
        for _ in range(2):
            d = dict(wl.x)
            d.update({k: torch.empty_like(wl.x[k]) for k in names})
            dev_in.append(d)
        o_dev = [wl.o, torch.empty_like(wl.o)]
        o_host = [torch.empty(wl.o.shape, dtype=wl.o.dtype).pin_memory() for _ in range(2)]
        h2d = sum(host[k].numel() * host[k].element_size() for k in names)
        d2h = o_host[0].numel() * o_host[0].element_size()
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        computed = [torch.cuda.Event() for _ in range(2)]
        drained = [torch.cuda.Event() for _ in range(2)]
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        e_start.record(stream)
        up.wait_event(e_start)
        for i in range(args.steps):
            j = i % 2
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(computed[j])       # step i-2 has read dev_in[j]
                for k in names:
                    dev_in[j][k].copy_(host[k], non_blocking=True)
                copied[j].record(up)
            stream.wait_event(copied[j])
            if i >= 2:
                stream.wait_event(drained[j])        # step i-2's result has left o_dev[j]
            wl.o = o_dev[j]
            wl.step(dev_in[j])
            computed[j].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(computed[j])
                o_host[j].copy_(o_dev[j], non_blocking=True)
                drained[j].record(down)
        for j in range(2):
            stream.wait_event(drained[j])
        e_end.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        wl.o = o_dev[0]
        e_s = max_over_ranks(e_start.elapsed_time(e_end)) / args.steps / 1e3
        if isinstance(wl, Prefill):
            e2e = {"value": weak_scaling_throughput(wl.units, world, e_s), "unit": "tok/s"}
        else:
            e2e = {"value": weak_scaling_throughput(wl.bytes, world, e_s) / 1e9, "unit": "GB/s"}
        e2e.update({"h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h})

    if rank == 0:
        hbm_peak, bf16_peak, peak_kind = measured_peaks()
        src = "MEASURED_PEAKS.json" if peak_kind == "measured" else "fallback"
        if isinstance(wl, Prefill):
            value = weak_scaling_throughput(wl.units, world, ms_per_step / 1e3)
            unit = "tok/s"
            # dominant phase: the scan is tensor-core work against the tf32 peak (the measured
            # bf16 peak times the nominal tf32 / bf16 ratio); the prepare phase is fp32 FMA work
            # against 148 SMs x 128 lanes x 2 flop x the maximum SM clock
            k = max(range(nph), key=lambda j: phase_ms[j])
            achieved = wl.phase_work[k] / (phase_ms[k] / 1e3) / 1e12
            if wl.phase_names[k] == "scan":
                bound, peak = "tensor", bf16_peak * NOMINAL_TF32_OVER_BF16
                peak_source = "%s bf16_tflops x nominal tf32/bf16 (1.1/2.25), %s" % (src, peak_kind)
            else:
                bound, peak = "alu", 148 * 128 * 2 * 1965e6 / 1e12
                peak_source = "148 SMs x 128 fp32 lanes x 2 flop x 1965 MHz"
            roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                        "frac": achieved / peak, "peak_source": peak_source,
                        "traffic": ncu_traffic(name), "kernel": wl.phase_kernel[k],
                        "algorithmic_flops_per_launch": wl.phase_work[k],
                        "phase_ms": dict(zip(wl.phase_names, phase_ms)),
                        "phase_timing": "each phase over the whole prompt, one after the other, in a "
                                        "second loop of K steps (the timed step runs them in %d pieces, "
                                        "the scan of one beside the prepare of the next, on two streams)"
                                        % (wl.launches_per_step // 2)}
            # and the HBM side over the whole step: the minimum bytes (q, k, v read once, the
            # outputs written once, the final state) against the measured copy bandwidth
            w = wl.w
            el = 2 if w.in_dtype == "bf16" else 4
            min_bytes = (2 * w.B * w.T * w.H_k * w.d_k * el + w.B * w.T * w.H_v * w.d_v * el
                         + 2 * w.B * w.T * w.H_v * el + w.B * w.T * w.H_v * w.d_v * 4
                         + w.B * w.H_v * w.d_v * w.d_k * 4)
            hbm_gbs = min_bytes / (ms_per_step / 1e3) / 1e9
            roofline["hbm"] = {"achieved": hbm_gbs, "peak": hbm_peak, "unit": "GB/s", "frac": hbm_gbs / hbm_peak,
                               "min_bytes_per_step": min_bytes,
                               "note": "minimum bytes; the workspace (records and key/query tiles, ~3 GB "
                                       "written and read back per step) comes on top"}
            dtype = Prefill.dtype
        else:
            value = weak_scaling_throughput(wl.bytes, world, ms_per_step / 1e3) / 1e9
            unit = "GB/s"
            calls = getattr(wl, "calls_per_step", wl.launches_per_step)   # acceptance: one call, two kernels
            kernel_ms = local_ms / args.steps / calls   # average launch duration over the timed region
            per_launch_bytes = wl.bytes / calls
            achieved = per_launch_bytes / (kernel_ms / 1e3) / 1e9
            roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                        "frac": achieved / hbm_peak, "peak_source": "%s hbm_gbs (%s)" % (src, peak_kind),
                        "traffic": ncu_traffic(name),
                        "algorithmic_bytes_per_launch": per_launch_bytes}
            dtype = "f32"
        line = {
            "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
            "data": "synthetic", "config": dict(wl.config(), parallelism="dp%d" % world),
            "token_heads_per_s": wl.units * world / (ms_per_step / 1e3)
            if not isinstance(wl, Prefill) else None,
            "frac_of_spec_8TBps": (wl.bytes * world / (ms_per_step / 1e3) / 1e9 / world) / SPEC_HBM_GBS
            if not isinstance(wl, Prefill) else None,
            "roofline": roofline,
            "clocks": clk.summary(),
            "gpu_launches": args.steps * wl.launches_per_step,
            "e2e": e2e,
        }
        if not args.no_cpu_baseline and world == 1:
            per_unit, units, desc, threads = oracle_sample(name, cpu_budget_s)
            cv, cu = cpu_value(name, per_unit)
            line["cpu_baseline"] = {"value": cv, "unit": cu, "cores": threads, "kind": "oracle",
                                    "sample": desc}

    if isinstance(wl, (SingleSeq, ShortConv)):
        wl.graph = None
    return line if rank == 0 else None


# Workloads whose records the default run nests under "configs" beside the headline (batched
# verify): the other model-scale configurations, then the next rows built on the same path.
NESTED = ["decode", "prefill", "single_seq_verify", "commit_next_verify", "verify_gated",
          "short_conv", "accept", "accept_greedy"]
# keys of a nested record (the headline line carries the run-wide ones)
NESTED_KEYS = ["value", "unit", "ms_per_step", "dtype", "config", "token_heads_per_s", "frac_of_spec_8TBps",
               "roofline", "clocks", "gpu_launches", "e2e", "cpu_baseline"]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["all"] + sorted(WORKLOADS), default="all",
                    help="all (default): batched_verify as the headline, the others nested "
                         "under \"configs\"")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=0,
                    help="prefill only: prompt length override (default 32768), for profiling a "
                         "smaller case")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import datetime
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    Prefill.tokens = args.tokens
    if args.workload != "all":
        line = measure(args.workload, args, rank, world, dev, barrier, 10.0)
    else:
        line = measure("batched_verify", args, rank, world, dev, barrier, 10.0)
        nested = {}
        for name in NESTED:
            torch.cuda.empty_cache()
            rec = measure(name, args, rank, world, dev, barrier, 1.5)
            if rank == 0:
                nested[name] = {k: rec[k] for k in NESTED_KEYS if k in rec}
        if rank == 0:
            line["configs"] = nested
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
