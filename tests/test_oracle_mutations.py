"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that
the pins in test_oracle_pins.py catch every one of them.

Each mutant is compiled into a temporary directory and loaded through
MOE_ORACLE_LIB in a child pytest process; the real oracle is never touched.
"""
import os
import subprocess
import sys

import pytest

from oracle import build as obuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "silu_on_up_projection": ("g[c] = (g[c] / (1.0 + exp(-g[c]))) * u[c];",
                              "g[c] = g[c] * (u[c] / (1.0 + exp(-u[c])));"),
    "ties_to_higher_index": ("return (x->idx < y->idx) ? -1 : (x->idx > y->idx);",
                             "return (x->idx > y->idx) ? -1 : (x->idx < y->idx);"),
    "capacity_floor": ("C = (long long)ceil(", "C = (long long)floor("),
    "bias_in_weights": ("ssum += (double)s[oi[j]];", "ssum += (double)u[oi[j]];"),
    "group_score_top1": ("for (int i = 1; i < group_score_topk; ++i)",
                         "for (int i = 1; i < 1; ++i)"),
    "down_projection_transposed": ("y[o] += g[c] * ld(W2, w_dtype, (size_t)c * d + o);",
                                   "y[o] += g[c] * ld(W2, w_dtype, (size_t)o * f + c);"),
    "renorm_missing": ("ow[j] = (exp((double)l[oi[j]] - m) / z) / psel;",
                       "ow[j] = (exp((double)l[oi[j]] - m) / z);"),
    "no_capacity": ("kept[e] = (C >= 0 && counts[e] > C) ? (int)C : counts[e];",
                    "kept[e] = counts[e];"),
    "logit_bias_sign": ("if (logit_bias) acc += (double)logit_bias[e];",
                        "if (logit_bias) acc -= (double)logit_bias[e];"),
    "shared_expert_dropped": ("for (int c = 0; c < d; ++c) o[c] += y[c];",
                              "for (int c = 0; c < d; ++c) o[c] += 0.0 * y[c];"),
    "exp_lo_term_missing": ("r = fmaf(-n, OR_LN2_LO, r);", "r = r;"),
    "e4m3_ties_away_from_zero": ("if (rem > 0.5 || (rem == 0.5 && fmod(n, 2.0) == 1.0)) n += 1.0;",
                                 "if (rem >= 0.5) n += 1.0;"),
    "e4m3_exponent_bias_8": ("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)"),
    "fp8_scale_for_e5m2_range": ("amax / 448.0f : 1.0f", "amax / 57344.0f : 1.0f"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation site not unique: {old}"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", *obuild.CFLAGS, "-o", str(lib), str(mpath), "-lm"])
    env = dict(os.environ, MOE_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 1, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
