"""The oracle pins must bite: each planted mistake in a copy of the oracle fails them.

Mistakes are planted in a temporary copy of ``oracle/nq_oracle.c`` on the CPU (never in the
CUDA path); the pin suite then runs against that copy in a subprocess and must fail.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "nq_oracle.c")

MUTATIONS = [
    # Gram from popcount: a dropped factor of 2
    ("return (int32_t)(r - 2 * differ);", "return (int32_t)(r - differ);"),
    # a dropped s2 term in the materialised weight
    ("double w = s1 * (double)gram_entry_packed(U + i * ldu, V + j * ldv, r) * s2[j];",
     "double w = s1 * (double)gram_entry_packed(U + i * ldu, V + j * ldv, r);"),
    # a wrong sign in the factored stage 1
    ("t[k] += bit ? z : -z;", "t[k] += bit ? z : z;"),
    # a transposed operand: V indexed by the output row
    ("double w = s1 * (double)gram_entry_packed(U + i * ldu, V + j * ldv, r) * s2[j];",
     "double w = s1 * (double)gram_entry_packed(U + (j % d_out) * ldu, V + (i % d_in) * ldv, r) * s2[j];"),
    # sign(0) read as -1
    ("if (v >= 0.0f) row", "if (v > 0.0f) row"),
    # MSB-first bit order
    ("row[k / 32] |= 1u << (k % 32);", "row[k / 32] |= 1u << (31 - k % 32);"),
    # bf16 rounding keeps one bit too few
    ("int qexp = e - 8;", "int qexp = e - 9;"),
    # fp16 decode with the wrong exponent bias
    ("v = ldexp((double)(1024 + f), e - 25);", "v = ldexp((double)(1024 + f), e - 24);"),
]

# mistakes in the calibration products, caught by their own pins
CAL = "test_oracle_calibration.py"
MUTATIONS += [
    # transpose: a dropped s2
    ("double w = s1[i] * (double)gram_entry_packed(U + i * ldu, V + j * ldv, r) * s2;",
     "double w = s1[i] * (double)gram_entry_packed(U + i * ldu, V + j * ldv, r);", CAL),
    # transpose: the cotangent read at the wrong row
    ("double term = w * yb[b * d_out + i];", "double term = w * yb[b * d_out + (d_out - 1 - i)];", CAL),
    # dL/ds1: a dropped s2
    ("double t1 = yb[b * d_out + i] * g * s2 * x[b * d_in + j];",
     "double t1 = yb[b * d_out + i] * g * x[b * d_in + j];", CAL),
    # dL/ds2: s2 where s1 belongs
    ("double t2 = x[b * d_in + j] * g * s1 * yb[b * d_out + i];",
     "double t2 = x[b * d_in + j] * g * s2 * yb[b * d_out + i];", CAL),
]
CONV = "test_oracle_converter.py"
MUTATIONS += [
    # balancing with the norm ratio inverted
    ("const double eta = (nu > 0.0 && nv > 0.0) ? sqrt(nv / nu) : 1.0;",
     "const double eta = (nu > 0.0 && nv > 0.0) ? sqrt(nu / nv) : 1.0;", CONV),
    # mean of the signed values instead of their magnitudes
    ("            acc += fabs(b);\n            if (b >= 0.0) U", "            acc += b;\n            if (b >= 0.0) U", CONV),
    # the mean divided by the row count instead of the row length
    ("if (s1_out) s1_out[i] = acc / (double)r;\n        s1_f16[i] = nq_oracle_double_to_f16(acc / (double)r);",
     "if (s1_out) s1_out[i] = acc / (double)d_out;\n        s1_f16[i] = nq_oracle_double_to_f16(acc / (double)d_out);",
     CONV),
    # fp16 encoder with the exponent field one too large
    ("return sign | (uint16_t)((e2 + 14) << 10) | frac;", "return sign | (uint16_t)((e2 + 15) << 10) | frac;", CONV),
]
SGR = "test_oracle_sign_grads.py"
MUTATIONS += [
    # dL/dU: a dropped s1
    ("double term = yb[b * d_out + i] * s1 * (double)sign_of_packed(V + j * ldv, k) *",
     "double term = yb[b * d_out + i] * (double)sign_of_packed(V + j * ldv, k) *", SGR),
    # dL/dV: the neighbouring rank column of U
    ("double term = x[b * d_in + j] * s2 * (double)sign_of_packed(U + i * ldu, k) *",
     "double term = x[b * d_in + j] * s2 * (double)sign_of_packed(U + i * ldu, (k + 1) % r) *", SGR),
    # the packed bits read as 0/1 instead of -1/+1
    ("return ((row[k / 32] >> (k % 32)) & 1u) ? 1 : -1;", "return ((row[k / 32] >> (k % 32)) & 1u) ? 1 : 0;", SGR),
]
MUTATIONS = [m if len(m) == 3 else (m[0], m[1], "test_oracle.py") for m in MUTATIONS]


@pytest.mark.parametrize("old,new,pins", MUTATIONS)
def test_pins_fail_on_planted_mistake(tmp_path, old, new, pins):
    src = open(SRC).read()
    assert old in src, "mutation anchor not found"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new, 1))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-o", str(so), str(mutant), "-lm"])
    env = dict(os.environ, NQ_ORACLE_SO=str(so))
    proc = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                           os.path.join(ROOT, "tests", pins)],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert proc.returncode != 0, "pins passed on a planted mistake: " + new
