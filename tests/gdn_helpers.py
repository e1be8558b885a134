"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI and the
oracle on the same seeded inputs, and compare with the max-abs-normalised error."""
import numpy as np
import torch

from gated_deltanet_mixer_verify_b200.inputs import as_f64, make_inputs, workload
from oracle import gdn_oracle as orc

# Tolerances (max |gpu - oracle| / max |oracle| per tensor): fp32 verify / decode outputs
# and state; prefill; bf16-stored outputs (8-bit mantissa, relative rounding 2^-9).
TOL = 1e-4
TOL_PREFILL = 2e-3
TOL_BF16_OUT = 8e-3


def rel_err(x, ref) -> float:
    x = x.detach().double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.max(np.abs(ref)) if ref.size else 1.0
    return float(np.max(np.abs(x - ref)) / max(den, 1e-300)) if ref.size else 0.0


def to_dev(x: dict, dev="cuda") -> dict:
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def oracle_verify(x: dict, accept_len, l2_eps=1e-6, scale=1.0):
    f = as_f64(x)
    L = None if accept_len is None else np.asarray(accept_len, dtype=np.int32)
    return orc.verify(f["q"], f["k"], f["v"], f["a"], f["b"], f["A_log"], f["dt_bias"], f["S0"],
                      L, l2_eps=l2_eps, scale=scale)


def gpu_verify(gdn, xd: dict, accept_len, inplace=True, out_dtype=torch.float32, scale=1.0,
               status=None, stash=None):
    state = xd["S0"].clone()
    out = state if inplace else torch.full_like(state, float("nan"))
    L = None if accept_len is None else torch.as_tensor(np.asarray(accept_len, np.int32)).cuda()
    o = gdn.verify_step(xd["q"], xd["k"], xd["v"], xd["a"], xd["b"], xd["A_log"], xd["dt_bias"],
                        state, out, L, stash=stash, scale=scale, status_word=status,
                        out_dtype=out_dtype)
    torch.cuda.synchronize()
    return o, out


# Runtime and profiler records a CUDA trace may hold besides kernels.
_NOT_KERNELS = ("cuda", "Activity Buffer Request")


def launched_kernels(fn):
    """Run fn and return (its result, the names of the CUDA kernels it launched), from the
    CUPTI kernel trace that torch.profiler collects. Once in a long run the trace held the
    runtime calls but no kernel record at all; fn cannot simply run again (many calls update
    a state in place), so then the name comes from the library's own record of the kernel its
    last verify or decode call chose (gdn_last_verify_kernel)."""
    from torch.profiler import ProfilerActivity, profile
    from gated_deltanet_mixer_verify_b200 import gdn
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        r = fn()
        torch.cuda.synchronize()
    names = {e.name for e in prof.events()}
    if not any(not n.startswith(_NOT_KERNELS) for n in names):
        names.add(gdn.last_verify_kernel())
    return r, names


def sm_count() -> int:
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
