"""Pin sensitivity: each plausible mistake planted in a copy of the oracle's C source must
make at least one pin fail (or the mutant crash). The product oracle is never modified; the
mutants are compiled into a temporary directory and run in a subprocess."""
import json
import os
import subprocess
import sys

import pytest

import oracle
from tests_support import ROOT

MUTANTS = {
    "drop_zero_point": ("return (q - z) * s;", "return q * s;"),
    "zero_sign": ("return (q - z) * s;", "return (q + z) * s;"),
    "scale_group_index": ("(size_t)(c / ORACLE_GROUP);\n    double s",
                          "(size_t)(c % ORACLE_GROUP);\n    double s"),
    "bit_order_in_byte": (">> (pos & 7)) & 1u)", ">> (7 - (pos & 7))) & 1u)"),
    "group_block_4bit_only": ("* 8 * bits;", "* 8 * 4;"),
    "silu_sign": ("g / (1.0 + exp(-g))", "g / (1.0 + exp(g))"),
    "silu_dropped": ("double silu = g / (1.0 + exp(-g));", "double silu = g;"),
    "tie_break_higher_index": ("l[e] > l[best]", "l[e] >= l[best]"),
    "softmax_unnormalised": ("wt[i] = exp(l[it[i]] - lmax) / den;", "wt[i] = exp(l[it[i]]) / den;"),
    "bias_dropped": ("if (bias) acc += (double)bias[e];", ""),
    "down_transposed": ("oracle_weight(ex, 2, H, I, r, c)", "oracle_weight(ex, 2, H, I, c % I, r % I)"),
    "gate_reads_up": ("g += oracle_weight(ex, 0,", "g += oracle_weight(ex, 1,"),
    "combine_weight_dropped": ("o[r] += wi * y[r];", "o[r] += y[r];"),
    "f16_exponent_bias": ("ex - 25)", "ex - 24)"),
    "f16_subnormal_scale": ("ldexp((double)man, -24)", "ldexp((double)man, -14)"),
    "router_reads_transposed": ("(double)wr[(size_t)e * H + h]", "(double)wr[(size_t)h * E + e]"),
    # quantiser
    "f16_round_truncates": ("double n = rint(ldexp(a, -qe));", "double n = floor(ldexp(a, -qe));"),
    "f16_subnormal_quantum": ("if (qe < -24) qe = -24;", "if (qe < -14) qe = -14;"),
    "hqq_levels_not_minus_one": ("double qmax = (double)((1 << bits) - 1);\n    double lo",
                                 "double qmax = (double)(1 << bits);\n    double lo"),
    "hqq_zero_from_max": ("double z = -lo / s;", "double z = -hi / s;"),
    "hqq_no_clamp": ("return fmin(fmax(q, 0.0), qmax);", "return q;"),
    "hqq_err_signed": ("err += fabs(w[j] - r[j]);", "err += w[j] - r[j];"),
    "hqq_shrink_exponent": ("pow(a, p - 1.0) / beta", "pow(a, p) / beta"),
    "hqq_shrink_beta_inverted": ("pow(a, p - 1.0) / beta", "pow(a, p - 1.0) * beta"),
    "hqq_zero_update_sign": ("acc += q[j] - (w[j] - e) / s;", "acc += q[j] + (w[j] - e) / s;"),
    "hqq_shrink_ignored": ("acc += q[j] - (w[j] - e) / s;", "acc += q[j] - w[j] / s;"),
    "hqq_beta_not_grown": ("beta *= kappa;", ""),
    "hqq_keeps_last_zero": ("oracle_f64_to_f16(fmin(fmax(zbest,", "oracle_f64_to_f16(fmin(fmax(z,"),
    "hqq_no_stop": ("if (!(err < best * HQQ_FALL)) break;", "if (!(err < best * HQQ_FALL)) continue;"),
    "hqq_strict_stop": ("if (!(err < best * HQQ_FALL)) break;", "if (!(err < best)) break;"),
    "hqq_codes_unrounded_zero": ("hqq_code(w[j], s, zs, qmax)", "hqq_code(w[j], s, zbest, qmax)"),
    "hqq_matrix_group_column": ("c0 = (g % gpr) * ORACLE_GROUP;", "c0 = (g / rows) * ORACLE_GROUP;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    msrc = tmp_path / "mutant.c"
    msrc.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    oracle.build(str(msrc), str(lib))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "oracle_pins.py"), str(lib)],
                       capture_output=True, text=True, timeout=300,
                       env={**os.environ, "OMP_NUM_THREADS": "2"})
    if r.returncode != 0:
        return  # the mutant crashed: caught
    res = json.loads(r.stdout.strip().splitlines()[-1])
    failed = [k for k, v in res.items() if v != "ok"]
    assert failed, f"no pin catches mutant {name}"
