"""CPU tests: plant one plausible mistake at a time in a copy of the oracle
source and check that at least one pin fails for each.  The built oracle itself
is never modified."""
import os
import shutil

import numpy as np
import pytest

import oracle
from tests import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "fa_oracle.c")

# (name, text in fa_oracle.c, replacement, how many occurrences to replace)
MUTANTS = [
    ("dk_drops_scale", "dkj[t] += pb->scale * ds * qi[t];", "dkj[t] += ds * qi[t];", None),
    ("dq_drops_scale", "dqi[t] += pb->scale * ds * kvec[t];", "dqi[t] += ds * kvec[t];", None),
    ("causal_offset_sign", "return j <= i + (pb->Nk - pb->Nq);",
     "return j <= i - (pb->Nk - pb->Nq);", None),
    ("causal_strict", "return j <= i + (pb->Nk - pb->Nq);", "return j < i + (pb->Nk - pb->Nq);",
     None),
    ("o_uses_k", """load_vec(pb->v, pb->dtype, kv_off(pb, b, g, j), d, kvec);
        for (int64_t t = 0; t < d; ++t)
            o_row[t] += p[j] * kvec[t];""", """load_vec(pb->k, pb->dtype, kv_off(pb, b, g, j), d, kvec);
        for (int64_t t = 0; t < d; ++t)
            o_row[t] += p[j] * kvec[t];""", None),
    ("online_no_rescale_U", "U[t] = a * U[t];", "U[t] = U[t];", None),
    ("online_no_rescale_l", "l = a * l;", "l = l;", None),
    ("ds_sign", "double ds = p[j] * (dp[j] - D);", "double ds = p[j] * (dp[j] + D);", None),
    ("gqa_modulo", "const int64_t g = h / (pb->Hq / pb->Hkv);", "const int64_t g = h % pb->Hkv;",
     None),
    ("lse_drops_log", "*lse_out = m + log(l);", "*lse_out = m + l;", None),
    ("dv_uses_ds", "dvj[t] += p[j] * doi[t];", "dvj[t] += ds * doi[t];", None),
    ("merge_weight_wrong_ref", "double w = exp(lse_parts[s] - L);",
     "double w = exp(lse_parts[s] - mx);", None),
    ("scale_squared", "s[j] = pb->scale * acc;", "s[j] = pb->scale * pb->scale * acc;", None),
    ("dq_transposed_operand", "dqi[t] += pb->scale * ds * kvec[t];",
     "dqi[t] += pb->scale * ds * qi[t];", None),
    ("e4m3_bias_8", "mag = ldexp(1.0 + m / 8.0, e - 7);", "mag = ldexp(1.0 + m / 8.0, e - 8);", None),
    ("e4m3_subnormal_step", "mag = ldexp((double)m, -9);", "mag = ldexp((double)m, -10);", None),
    ("e4m3_mantissa_width", "mag = ldexp(1.0 + m / 8.0, e - 7);", "mag = ldexp(1.0 + m / 16.0, e - 7);",
     None),
    ("e4m3_no_nan", "if (e == 15 && m == 7)", "if (e == 16)", None),
]


@pytest.mark.parametrize("name,old,new,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new, count):
    text = open(SRC, encoding="utf-8").read()
    assert old in text, f"mutation anchor for {name} not found"
    mutated = text.replace(old, new) if count is None else text.replace(old, new, count)
    src = tmp_path / "fa_oracle_mutant.c"
    src.write_text(mutated, encoding="utf-8")
    so = oracle.build_variant(str(src), str(tmp_path / "libmutant.so"))
    failed = []
    # a mutant may produce NaN or inf; the pins' assertions judge that, not numpy warnings
    with oracle.using(so), np.errstate(all="ignore"):
        for pin in P.ALL_PINS:
            try:
                pin()
            except AssertionError:
                failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
