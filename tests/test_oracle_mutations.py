"""Strength of the oracle's pins, on the CPU (no GPU needed).

Each case below plants one plausible mistake in a copy of the C oracle
(``oracle/lbca_oracle.c``), builds it, and runs the pin tests of the part it
touches against that build, with the agreement-with-brute-force tests left
out: the closed forms, special cases and invariants alone must reject it (a
mistake shared by the oracle and the NumPy brute force, both written from the
same reading of the pages, would pass the agreement tests).  A control build of
the unchanged source passes the same runs, so a failure is the mistake's.

The mistakes follow the method's steps: the visible-block count P(L)
("mSeek" README, "How LBCA works"), RMSNorm and RoPE of entries and queries
and the shared form's output turned back by -t (CSA page, "What is
implemented" and "Deviations from paper"), the pooling softmax over Z + B_pos
(HCA page, "What is implemented", Eqs 20-23), the sink in the denominator
only, the window start, the GQA head map and the softmax scale; CSA dual
pooling, the indexer's ReLU and mask, the sparse window (CSA page, Eqs 9-19);
and the terms of the backward pass (checked against finite differences).
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "lbca_oracle.c")
FWD = "tests/test_oracle_pins.py"
CSA = "tests/test_csa_oracle.py"
BWD = "tests/test_backward_oracle.py"

# name: (pin file, [(text, replacement, occurrences)])
MUTATIONS = {
    # P(L) = floor((L - w) / m) rounded the other way at the block edge
    "visible_count_shifted": (FWD, [("return p / m;", "return (p + 1) / m;", 1)]),
    "rmsnorm_eps_dropped": (FWD, [("double inv = 1.0 / sqrt(ss / D + eps);", "double inv = 1.0 / sqrt(ss / D);", 1)]),
    "rmsnorm_gain_dropped": (FWD, [("x[d] = x[d] * inv * (gamma ? gamma[d] : 1.0);", "x[d] = x[d] * inv;", 1)]),
    "rope_sign": (FWD, [("x[base + 2 * k] = a * cs - b * sn;", "x[base + 2 * k] = a * cs + b * sn;", 1)]),
    "rope_frequency": (FWD, [("pow(theta, -2.0 * k / rho)", "pow(theta, -1.0 * k / rho)", 1)]),
    "rope_leading_dims": (FWD, [("int base = D - rho;", "int base = 0;", 1)]),
    # B_pos indexed from the block's end (a transposed bias)
    "pool_bias_rows_reversed": (FWD, [("bpos[i * ts + (long)g * D + ch]", "bpos[(m - 1 - i) * ts + (long)g * D + ch]",
                                       2)]),
    "pool_key_rope_at_block_end": (FWD, [("(double)(pos0 + j * m));", "(double)(pos0 + j * m + m - 1));", 1)]),
    "sink_dropped": (FWD, [("/* one softmax over all scores plus the sink (denominator only) */\n"
                            "        double den = sink ? exp(sink[h] - smax) : 0.0;",
                            "/* one softmax over all scores plus the sink (denominator only) */\n"
                            "        double den = 0.0;", 1)]),
    "window_start_shifted": (FWD, [("const long s0 = P * m;", "const long s0 = P * m + 1;", 1)]),
    "head_map": (FWD, [("const int g = h / r;", "const int g = h % G;", 2)]),
    "scale": (FWD, [("1.0 / sqrt((double)D)", "1.0 / (double)D", 3)]),
    "shared_output_not_turned_back": (FWD, [("if (c->shared_kv && c->rope_dims) rope(o, D, c->rope_dims, "
                                             "c->rope_theta, -(double)t);", ";", 1)]),
    "query_rope_position": (FWD, [("rope(qt, D, c->rope_dims, c->rope_theta, (double)t);",
                                   "rope(qt, D, c->rope_dims, c->rope_theta, (double)(t + 1));", 3)]),
    "value_from_keys": (FWD, [("const double* val = v + (b * T_hist + s) * ts + (long)g * D;",
                               "const double* val = k + (b * T_hist + s) * ts + (long)g * D;", 1)]),
    "dual_b_bias_is_a_bias": (CSA, [("bpos_b[r * ts + col]", "bpos_a[r * ts + col]", 2)]),
    "dual_b_block_not_preceding": (CSA, [("(i - 1) * m + r", "i * m + r", 3)]),
    "dual_key_rope_position": (CSA, [("finalise_key(c, e, gamma, (double)(i * m));",
                                      "finalise_key(c, e, gamma, (double)((i + 1) * m));", 1)]),
    "indexer_relu_dropped": (CSA, [("(dot > 0.0 ? dot : 0.0)", "dot", 1)]),
    "indexer_mask_off_by_one": (CSA, [("if (j >= nvis[b]) {", "if (j > nvis[b]) {", 1)]),
    "sparse_window_short": (CSA, [("const long s0 = lens[b] - w > 0 ? lens[b] - w : 0;",
                                   "const long s0 = lens[b] - w + 1 > 0 ? lens[b] - w + 1 : 0;", 1)]),
    "sparse_output_not_turned_back": (CSA, [("if (c->rope_dims) rope(o, D, c->rope_dims, c->rope_theta, "
                                             "-(double)t);", ";", 1)]),
    "bwd_rmsnorm_power": (BWD, [("- x[d] * r * r * r * dot / D", "- x[d] * r * r * dot / D", 1)]),
    "bwd_softmax_centering_dropped": (BWD, [("const double dS = sc[e] * (dp - Dsum);",
                                             "const double dS = sc[e] * dp;", 1)]),
    "bwd_sink_sign": (BWD, [("ds[h] += -psink * Dsum;", "ds[h] += psink * Dsum;", 1)]),
    "bwd_pool_logit_uncentered": (BWD, [("const double da = wi * (x[tok] - Pc) * dPc;",
                                         "const double da = wi * x[tok] * dPc;", 1)]),
    "bwd_query_rope_turned_forward": (BWD, [("rope(dqt, D, c->rope_dims, c->rope_theta, -(double)t);",
                                             "rope(dqt, D, c->rope_dims, c->rope_theta, (double)t);", 1)]),
    "bwd_pool_weight_on_x": (BWD, [("gX[(long)sr * nx + tok] += wi * dPc;", "gX[(long)sr * nx + tok] += dPc;", 1)]),
}


def _build(text, path):
    with open(path + ".c", "w") as f:
        f.write(text)
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math", path + ".c",
                           "-o", path + ".so", "-lm"])
    return path + ".so"


def _pins(lib, pin_file):
    """Exit code of the pin file (brute-force agreement left out) on `lib`."""
    env = dict(os.environ, LBCA_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", pin_file, "-k", "not brute_force"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, (r.stdout + r.stderr)[-2000:]


@pytest.fixture(scope="module")
def runs(tmp_path_factory):
    """Every mutant's pin run and the control runs, four at a time."""
    d = str(tmp_path_factory.mktemp("mutants"))
    src = open(SRC).read()
    jobs = {("control", f): (_build(src, os.path.join(d, "control")), f) for f in (FWD, CSA, BWD)}
    for name, (pin_file, edits) in MUTATIONS.items():
        text = src
        for old, new, n in edits:
            assert text.count(old) == n, f"{name}: the oracle source no longer has {n} x {old!r}"
            text = text.replace(old, new)
        jobs[(name, pin_file)] = (_build(text, os.path.join(d, name)), pin_file)
    with ThreadPoolExecutor(max_workers=4) as ex:
        futs = {k: ex.submit(_pins, *v) for k, v in jobs.items()}
        return {k: f.result() for k, f in futs.items()}


@pytest.mark.parametrize("pin_file", [FWD, CSA, BWD])
def test_unchanged_oracle_passes_the_pins(runs, pin_file):
    rc, tail = runs[("control", pin_file)]
    assert rc == 0, tail


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_planted_mistake_fails_a_pin(runs, name):
    pin_file = MUTATIONS[name][0]
    rc, tail = runs[(name, pin_file)]
    # 1: a pin failed; < 0: the mutant itself crashed (a window that comes out
    # shorter than the arrays sized from it).  Usage or collection errors do not count.
    assert rc == 1 or rc < 0, f"{name}: pin run of {pin_file} ended with {rc}:\n{tail}"
