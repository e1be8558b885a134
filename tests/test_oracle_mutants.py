"""Plant plausible mistakes in copies of the oracle's C source and check that the pins in
test_oracle*.py catch every one (a dropped term, a wrong sign or index,
a transposed operand, an off-by-one commit, reversed filter taps, a history not rewound). Mistakes are planted only in the oracle, on the CPU."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gdn_oracle.c")

MUTANTS = {
    "beta_term_sign": ("al * (s - be * p[i] * kt[j])", "al * (s + be * p[i] * kt[j])"),
    "alpha_dropped": ("al * (s - be * p[i] * kt[j])", "(s - be * p[i] * kt[j])"),
    "alpha_on_write": ("+ be * vt[i] * kt[j];", "+ al * be * vt[i] * kt[j];"),
    "output_transposed": ("acc += S[(int64_t)i * dk + j] * qt[j];",
                          "acc += S[(int64_t)j * dk + i] * qt[j];"),
    "key_for_query_in_read": ("acc += S[(int64_t)i * dk + j] * qt[j];",
                              "acc += S[(int64_t)i * dk + j] * kt[j];"),
    "query_for_key_in_delta": ("acc += S[(int64_t)i * dk + j] * kt[j];",
                               "acc += S[(int64_t)i * dk + j] * qt[j];"),
    "gqa_modulo": ("const int g = h / G;\n            int L", "const int g = h % Hk;\n            int L"),
    "softplus_branch": ("fmax(x, 0.0) + log1p", "fmin(x, 0.0) + log1p"),
    "sigmoid_sign": ("1.0 / (1.0 + exp(-x))", "1.0 / (1.0 + exp(x))"),
    "eps_outside_sqrt": ("1.0 / sqrt(ss + eps)", "1.0 / (sqrt(ss) + eps)"),
    "scale_on_keys": ("oracle_l2norm(nk, dk, k, l2_eps, 1.0, kh)", "oracle_l2norm(nk, dk, k, l2_eps, scale, kh)"),
    "commit_off_by_one": ("if (t + 1 == L) memcpy", "if (t == L) memcpy"),
    "A_log_not_exponentiated": ("-exp(A_log[h]) * sp(", "-A_log[h] * sp("),
    "dt_bias_sign": ("sp(a[idx] + dt_bias[h])", "sp(a[idx] - dt_bias[h])"),
    "chunk_state_term_sign": ("U[t * dv + i] = Ut[t * dv + i] - ws;", "U[t * dv + i] = Ut[t * dv + i] + ws;"),
    "chunk_decay_reversed": ("beta[GI(t)] * exp(Gc[t] - Gc[s]) * kk", "beta[GI(t)] * exp(Gc[s] - Gc[t]) * kk"),
    "chunk_output_diag_dropped": ("for (int s = 0; s <= t; ++s) {\n                        double d = 0.0;",
                                  "for (int s = 0; s < t; ++s) {\n                        double d = 0.0;"),
    "chunk_handoff_decay_dropped": ("double acc = eglast * S[(int64_t)i * dk + j];",
                                    "double acc = S[(int64_t)i * dk + j];"),
    "conv_taps_reversed": ("z += w[(int64_t)c * K + i] * xc[t + i];",
                           "z += w[(int64_t)c * K + (K - 1 - i)] * xc[t + i];"),
    "conv_silu_dropped": ("* C + c] = z / (1.0 + exp(-z));", "* C + c] = z;"),
    "conv_history_not_rewound": ("const int from = ok ? L : 0;", "const int from = ok ? T : 0;"),
    "conv_history_transposed": ("for (int r = 0; r < H; ++r) xc[r] = hist[((int64_t)b * H + r) * C + c];",
                                "for (int r = 0; r < H; ++r) xc[r] = hist[(int64_t)b * H * C + (int64_t)c * H + r];"),
    "conv_bad_count_commits": ("const int from = ok ? L : 0;", "const int from = ok ? L : T;"),
    "norm_sum_not_mean": ("1.0 / sqrt(ss / d + eps);", "1.0 / sqrt(ss + eps);"),
    "norm_eps_outside_sqrt": ("1.0 / sqrt(ss / d + eps);", "1.0 / (sqrt(ss / d) + eps);"),
    "norm_gate_sigmoid_not_silu": ("const double g = zrow[j] / (1.0 + exp(-zrow[j]));",
                                   "const double g = 1.0 / (1.0 + exp(-zrow[j]));"),
    "norm_weight_dropped": ("y[r * d + j] = orow[j] * inv * w[j] * g;", "y[r * d + j] = orow[j] * inv * g;"),
    "norm_gate_on_wrong_row": ("const double* zrow = z + r * d;", "const double* zrow = z;"),
    "accept_ratio_inverted": ("ok = u[(int64_t)b * T + t + 1] * qv < pv;", "ok = u[(int64_t)b * T + t + 1] * pv < qv;"),
    "accept_residual_reversed": ("q[j] = fmax(p[j] - q[j], 0.0);", "q[j] = fmax(q[j] - p[j], 0.0);"),
    "accept_len_without_anchor": ("accept_len[b] = n + 1;", "accept_len[b] = n;"),
    "accept_greedy_tie_to_last": ("if (lt[j] > lt[am]) am = j;", "if (lt[j] >= lt[am]) am = j;"),
    "accept_next_from_previous_row": ("const double* ln = target + ((int64_t)b * T + n) * V;",
                                      "const double* ln = target + ((int64_t)b * T + (n > 0 ? n - 1 : 0)) * V;"),
    "accept_temperature_ignored": ("for (int j = 0; j < V; ++j) p[j] = exp((l[j] - m) / tau) / s;",
                                   "for (int j = 0; j < V; ++j) p[j] = exp(l[j] - m) / s;"),
    "accept_continues_after_rejection": ("if (!stopped && ok) {", "if (ok) {"),
}


def pin_file(name):
    """The pins of the function a mutant breaks: conv_* the short convolution's, norm_* the
    gated normalisation's, accept_* the acceptance's, the rest the mixer's."""
    if name.startswith("conv_"):
        return "test_oracle_conv.py"
    if name.startswith("norm_"):
        return "test_oracle_norm.py"
    if name.startswith("accept_"):
        return "test_oracle_accept.py"
    return "test_oracle.py"


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, "mutation anchor not found: " + name
    mutated = src.replace(old, new, 1)
    c = tmp_path / "mut.c"
    c.write_text(mutated)
    lib = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(lib),
                    str(c), "-lm"], check=True)
    env = dict(os.environ, GDN_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", pin_file(name))],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, "pins did not catch mutant %s:\n%s" % (name, r.stdout[-2000:])
