"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of moe_oracle.c (on the CPU), builds it, and
runs the pin suites (test_oracle_pins.py, test_oracle_cache_route.py) against that build
in a child process: the suites have to fail.
"""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTANTS = {
    "silu_sign": ("hbuf[i] = a / (1.0 + exp(-a)) * u;", "hbuf[i] = a / (1.0 + exp(a)) * u;"),
    "shared_term_dropped": ("o[h] += s[t] * y[h];", "o[h] += 0.0 * y[h];"),
    "down_transposed": ("acc += w_at(wd, sd, dtype, I, h, i) * hbuf[i];",
                        "acc += w_at(wd, sd, dtype, I, i, h) * hbuf[i];"),
    "tie_to_higher_id": ("if (best < 0 || l[e] > l[best])", "if (best < 0 || l[e] >= l[best])"),
    "no_renormalisation": ("w[(long)t * k + j] = p[id[j]] / ps;", "w[(long)t * k + j] = p[id[j]];"),
    "bias_ignored": ("acc += (double)L->router_bias[e];", "acc += 0.0;"),
    "nibble_order": ("int nibble = (c & 1) ? (byte >> 4) : (byte & 15);",
                     "int nibble = (c & 1) ? (byte & 15) : (byte >> 4);"),
    "gate_up_swapped": ("a += w_at(wg, sg, dtype, H, i, h) * x[h];", "a += w_at(wu, su, dtype, H, i, h) * x[h];"),
    "shared_gate_sign": ("s[t] = 1.0 / (1.0 + exp(-gx));", "s[t] = 1.0 / (1.0 + exp(gx));"),
    "group_order_reversed": ("perm[cursor[ids[i]]++] = (int32_t)i;",
                             "perm[offsets[ids[i] + 1] - 1 - (cursor[ids[i]]++ - offsets[ids[i]])] = (int32_t)i;"),
    "renorm_not_renormalised": ("w[j] = (exp(logits_row[ids[j]] - m) / z) / ps;",
                                "w[j] = (exp(logits_row[ids[j]] - m) / z);"),
    "renorm_wrong_index": ("w[j] = (exp(logits_row[ids[j]] - m) / z) / ps;",
                           "w[j] = (exp(logits_row[j] - m) / z) / ps;"),
    "cache_weights_from_biased_logits": ("w[t * k + j] = (exp(z[id[j]] - zmax) / zsum) / ps;",
                                         "w[t * k + j] = (exp(zb[id[j]] - zmax) / zsum) / ps;"),
    "cache_delta_is_max_only": ("const double delta = zmax - zmin;", "const double delta = zmax;"),
    "cache_bias_sign": ("zb[e] = z[e] + lambda * delta * (cached[e] ? 1.0 : 0.0);",
                        "zb[e] = z[e] - lambda * delta * (cached[e] ? 1.0 : 0.0);"),
    "int2_code_order": ("int code = (byte >> (2 * (c % 4))) & 3;", "int code = (byte >> (6 - 2 * (c % 4))) & 3;"),
    "int2_code_offset": ("return group_scale(scale, K, n, c) * (double)(code - 2);",
                         "return group_scale(scale, K, n, c) * (double)(code - 1);"),
    "scale_group_index": ("return bf16_bits_to_double(scale[n * (K / 32) + c / 32]);",
                          "return bf16_bits_to_double(scale[n * (K / 32) + (c / 32 + 1) % (K / 32)]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutant_c = tmp_path / "mutant.c"
    mutant_c.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(mutant_c),
                           "-o", str(so), "-lm"])
    env = dict(os.environ, ORACLE_LIB=str(so), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                        os.path.join(ROOT, "tests", "test_oracle_cache_route.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutant {name}:\n{r.stdout[-2000:]}"
