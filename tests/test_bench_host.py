"""bench.py's host-side accounting, without a GPU: the stash size it charges matches the
library's own gdn_stash_bytes, the commit-on-next-verify byte count adds exactly the two
stashes and the state write-back of every sequence, and the reference arm (the oracle on the
host cores) prints one JSON line for the new workload."""
import importlib.util
import json
import os
import subprocess
import sys

import pytest

from gated_deltanet_mixer_verify_b200 import build as gbuild
from gated_deltanet_mixer_verify_b200.inputs import workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("T", [1, 5, 8])
def test_stash_floats_match_the_library(bench, T):
    gbuild.build()
    from gated_deltanet_mixer_verify_b200 import gdn
    assert bench.stash_floats_per_head(T, 128, 128) * 4 * 64 * 48 == gdn.stash_bytes(64, T, 16, 48, 128, 128)


def test_commit_next_bytes(bench):
    w = workload("batched_verify")
    state = w.B * w.H_v * w.d_v * w.d_k * 4
    stash = w.B * w.H_v * (w.T * w.d_k + 8 + w.T * w.d_v) * 4
    # the verify call's bytes with every sequence's state written back, plus two stashes
    assert bench.commit_next_bytes(w) == bench.algorithmic_bytes(w, n_state_writes=w.B) + 2 * stash
    assert bench.algorithmic_bytes(w, n_state_writes=w.B) - bench.algorithmic_bytes(w, n_state_writes=0) == state


def test_reference_arm_commit_next_verify():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "commit_next_verify", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["config"]["workload"] == "commit_next_verify"
    assert d["unit"] == "GB/s" and d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0


def test_conv_bytes(bench):
    w = workload("batched_verify")
    C = 2 * 16 * 128 + 48 * 128
    # q, k, v in and out (bf16), history in and out (3 rows), taps (fp32), accept counts
    assert bench.conv_bytes(w) == 2 * 64 * 8 * C * 2 + 2 * 64 * 3 * C * 2 + C * 4 * 4 + 64 * 4


def test_reference_arm_short_conv():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "short_conv", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    d = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][0])
    assert d["config"]["workload"] == "short_conv" and d["cpu_baseline"]["cores"] == 1 and d["value"] > 0


def test_gated_bytes_and_reference_arm(bench):
    w = workload("batched_verify")
    assert bench.gated_bytes(w) == bench.algorithmic_bytes(w) + 64 * 8 * 48 * 128 * 2 + 128 * 4
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "verify_gated", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    d = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][0])
    assert d["config"]["workload"] == "verify_gated" and d["value"] > 0


@pytest.mark.parametrize("name", ["accept", "accept_greedy"])
def test_accept_bytes_and_reference_arm(bench, name):
    w = workload("batched_verify")
    V = 151936
    sampled = name == "accept"
    expect = 64 * 8 * V * 2 + (64 * 7 * V * 2 if sampled else 0) + 64 * 8 * 4 + (64 * 8 * 4 if sampled else 0) + 2 * 64 * 4
    assert bench.accept_bytes(w, sampled) == expect
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", name, "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    d = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][0])
    assert d["config"]["workload"] == name and d["value"] > 0 and d["cpu_baseline"]["cores"] == 1


def test_default_reference_arm_times_the_headline_config():
    # the driver's reference call passes no --workload: the oracle runs on batched verify
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["config"]["workload"] == "batched_verify"


def test_nested_records_cover_the_model_scale_configs(bench):
    # the default run nests decode, prefill and the 48-layer single sequence beside the
    # headline, each record with its own timing, roofline, clocks and end-to-end leg
    assert bench.NESTED[:3] == ["decode", "prefill", "single_seq_verify"]
    assert set(bench.NESTED) | {"batched_verify"} == set(bench.WORKLOADS)
    for k in ("value", "unit", "ms_per_step", "roofline", "clocks", "e2e", "gpu_launches"):
        assert k in bench.NESTED_KEYS
    assert all(hasattr(bench.WORKLOADS[n], "e2e") or n in ("decode", "prefill", "accept", "accept_greedy",
                                                           "commit_next_verify", "verify_gated")
               for n in bench.NESTED)
