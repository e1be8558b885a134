"""Write the stored expected values under tests/golden/ from the fp64 oracle alone.

Run from the repository root:  python tests/golden/make_golden.py
Inputs come from the seeded generator; expected values come only from oracle/.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from gated_deltanet_mixer_verify_b200.inputs import as_f64, make_inputs, workload  # noqa: E402
from oracle import gdn_oracle as orc  # noqa: E402


def tiny_verify():
    w = workload("tiny_verify")
    x = as_f64(make_inputs(w))
    o, Sc, bad = orc.verify(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                            x["S0"], x["accept_len"], l2_eps=1e-6, scale=1.0)
    return {
        "source": "fp64 oracle (oracle/gdn_oracle.c) on the seeded tiny_verify workload: "
                  "B=1, H_k=H_v=2, d=16, T=8, fp32 inputs, l2_eps=1e-6, scale=1",
        "accept_len": [int(v) for v in x["accept_len"]],
        "o_shape": list(o.shape), "o": [float(v) for v in o.ravel()],
        "S_commit_shape": list(Sc.shape), "S_commit": [float(v) for v in Sc.ravel()],
    }


if __name__ == "__main__":
    path = os.path.join(HERE, "tiny_verify_oracle.json")
    with open(path, "w") as f:
        json.dump(tiny_verify(), f, indent=0)
    print("wrote", path)
