"""Planted mistakes: the oracle's pins must catch plausible errors.

Each case below plants one mistake in a copy of oracle/moe_oracle.c (a dropped
term, a wrong sign, index or operand, a rule applied where it must not be),
builds the copy with the same gcc flags, and runs the whole pin suite
(tests/test_oracle_pins.py) against it in a subprocess.  The case passes when
at least one pin fails on the mutant.  The oracle itself is never modified;
the copies live in a temporary directory.
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# (name, text in moe_oracle.c, replacement): every text occurs exactly once.
MUTANTS = [
    # router and scores
    ("router_reads_transposed_weights",
     "const uint16_t *w = Wr + (size_t)e * d;\n        for (int i = 0; i < d; ++i)\n"
     "            acc += bf16_to_double(x_t[i]) * bf16_to_double(w[i]);",
     "for (int i = 0; i < d; ++i)\n            acc += bf16_to_double(x_t[i]) * "
     "bf16_to_double(Wr[(size_t)i * E + e]);"),
    ("softmax_not_normalised", "for (int e = 0; e < E; ++e) s[e] /= z;", "(void)z;"),
    ("sigmoid_wrong_sign", "s[e] = 1.0 / (1.0 + exp(-logit[e]));", "s[e] = 1.0 / (1.0 + exp(logit[e]));"),
    ("sqrt_dropped_from_sqrt_softplus", "s[e] = sqrt(softplus(logit[e]));", "s[e] = softplus(logit[e]);"),
    ("softplus_without_linear_part", "return (z > 0.0 ? z : 0.0) + log1p(exp(-fabs(z)));",
     "return log1p(exp(-fabs(z)));"),
    # selection
    ("bias_also_applied_to_softmax",
     "const int use_bias = (J->bias != NULL) && (J->score_fn != ORACLE_SOFTMAX);",
     "const int use_bias = (J->bias != NULL);"),
    ("bias_ignored", "kv[e].key = s[e] + (use_bias ? (double)J->bias[e] : 0.0);", "kv[e].key = s[e];"),
    ("ties_to_higher_index", "return (a->idx < b->idx) ? -1 : (a->idx > b->idx);",
     "return (a->idx > b->idx) ? -1 : (a->idx < b->idx);"),
    ("picks_smallest_keys", "if (a->key > b->key) return -1;\n    if (a->key < b->key) return 1;",
     "if (a->key < b->key) return -1;\n    if (a->key > b->key) return 1;"),
    # weights
    ("bias_leaks_into_weights", "for (int j = 0; j < k; ++j) { w[j] = s[sel[j]]; denom += w[j]; }",
     "for (int j = 0; j < k; ++j) { w[j] = kv[j].key; denom += w[j]; }"),
    ("renormalisation_dropped", "if (J->norm_topk) {\n            if (denom < DBL_MIN)",
     "if (0) {\n            if (denom < DBL_MIN)"),
    ("route_scale_dropped", "for (int j = 0; j < k; ++j) w[j] *= J->route_scale;", "(void)0;"),
    ("renormalised_over_all_experts", "if (denom < DBL_MIN) denom = DBL_MIN;",
     "denom = 0.0; for (int e = 0; e < E; ++e) denom += s[e];"),
    # experts
    ("silu_wrong_sign", "h[j] = (g / (1.0 + exp(-g))) * u;", "h[j] = (g / (1.0 + exp(g))) * u;"),
    ("gate_and_up_swapped", "h[j] = (g / (1.0 + exp(-g))) * u;", "h[j] = (u / (1.0 + exp(-u))) * g;"),
    ("silu_replaced_by_identity", "h[j] = (g / (1.0 + exp(-g))) * u;", "h[j] = g * u;"),
    ("down_projection_transposed", "acc += bf16_to_double(dr[j]) * h[j];",
     "acc += bf16_to_double(D[(size_t)j * d + m]) * h[j];"),
    ("combine_weight_dropped", "y[m] += w * acc;", "y[m] += acc;"),
    ("shared_experts_dropped", "for (int sh = 0; sh < J->S; ++sh) {", "for (int sh = 0; sh < 0; ++sh) {"),
    ("shared_gate_wrong_sign", "gw = 1.0 / (1.0 + exp(-z));", "gw = 1.0 / (1.0 + exp(z));"),
    ("last_routed_expert_skipped",
     "for (int j = 0; j < k; ++j) {\n        const size_t e = (size_t)sel[j];",
     "for (int j = 0; j < k - 1; ++j) {\n        const size_t e = (size_t)sel[j];"),
    # RMSNorm prologue
    ("rmsnorm_gain_not_zero_centred", "rstd * (1.0 + bf16_to_double(gain[i]))", "rstd * bf16_to_double(gain[i])"),
    ("rmsnorm_sum_not_mean", "1.0 / sqrt(ss / d + eps)", "1.0 / sqrt(ss + eps)"),
    ("rmsnorm_eps_outside_root", "1.0 / sqrt(ss / d + eps)", "1.0 / (sqrt(ss / d) + eps)"),
    # rounding to bf16
    ("bf16_ties_away_from_zero", "double q = nearbyint(ldexp(a, -qe));", "double q = round(ldexp(a, -qe));"),
    ("bf16_truncates", "double q = nearbyint(ldexp(a, -qe));", "double q = floor(ldexp(a, -qe));"),
    ("bf16_flushes_subnormals", "if (qe < -133) qe = -133;", "if (e < -125) return sign;"),
    # FP8 weights
    ("e4m3_exponent_bias_8", "else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
     "else v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("e4m3_subnormal_scale", "if (e == 0) v = ldexp((double)m / 8.0, -6);",
     "if (e == 0) v = ldexp((double)m / 8.0, -7);"),
    ("e4m3_no_nan_code", "if (e == 15 && m == 7) return NAN;", "(void)0;"),
    ("mx_scales_row_major", "scale[((size_t)g * nb + c / 32) * rows + r]",
     "scale[((size_t)g * rows + r) * nb + c / 32]"),
    ("mx_scale_bias_off_by_one", "ldexp(1.0, (int)u - 127)", "ldexp(1.0, (int)u - 126)"),
]


def _run_mutant(tmpdir, name, old, new):
    src = open(SRC).read()
    if src.count(old) != 1:
        return name, "not applied", f"{src.count(old)} occurrences of the planted text"
    d = os.path.join(tmpdir, name)
    os.makedirs(d, exist_ok=True)
    mut_src = os.path.join(d, "moe_oracle.c")
    with open(mut_src, "w") as fh:
        fh.write(src.replace(old, new))
    lib = os.path.join(d, "liboracle.so")
    cc = subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", lib, mut_src, "-lm"],
                        capture_output=True, text=True)
    if cc.returncode != 0:
        return name, "build failed", cc.stderr[-2000:]
    env = dict(os.environ, MOE_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", PINS, "-x", "-q", "-p", "no:cacheprovider"],
                       capture_output=True, text=True, cwd=ROOT, env=env, timeout=600)
    tail = (r.stdout + r.stderr)[-1500:]
    return name, ("caught" if r.returncode == 1 and " failed" in r.stdout else f"rc={r.returncode}"), tail


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    tmp = str(tmp_path_factory.mktemp("oracle_mutants"))
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        futs = [ex.submit(_run_mutant, tmp, n, o, w) for n, o, w in MUTANTS]
        return {name: (status, tail) for name, status, tail in (f.result() for f in futs)}


def test_unmutated_copy_passes_every_pin(tmp_path):
    """The harness itself: an unchanged copy built the same way passes."""
    name, status, tail = _run_mutant(str(tmp_path), "identity", "int oracle_moe_forward(",
                                     "int oracle_moe_forward(")
    assert status == "rc=0", tail


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(mutant_results, name):
    status, tail = mutant_results[name]
    assert status == "caught", f"{name}: {status}\n{tail}"
