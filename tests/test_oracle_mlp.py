"""Pins for the oracle's MLP composition (``oracle.mlp``), CPU only.

The MLP block is not on the pages: it is how the 7B and 70B MLP workloads chain three LRB
layers (page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models",
section 2, factorisation equation, for each projection) with h = bf16(silu(g) * u) between
them.  The pins below hold it to values fixed without the oracle's own arithmetic:

* power-of-two scales and integer activations make every gate and up output a dyadic
  rational that numpy's integer matmul of the unpacked signs gives exactly;
* where bf16(g) >= 40, silu(g) = g to within 2^-57 relative, so h = bf16(bf16(g) bf16(u))
  unless that product sits exactly on a bf16 rounding midpoint; where bf16(g) <= -40,
  |h| <= 1e-15 |g u|; where g = 0, h = 0;
* with unit scales the down projection is numpy's matmul of its sign Gram matrix with h.

Together they catch an exchange of gate and up, a dropped bf16 rounding of g or of u, and a
down projection fed anything but h (the planted mistakes at the end).
"""
import os
import shutil
import subprocess
import sys

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

F16_ONE = 0x3C00       # 1.0
F16_EIGHTH = 0x3000    # 2^-3


def _signs(words, r):
    """Packed words [rows][ld] -> int64 signs [rows][r]: bit k % 32 of word k / 32, 1 -> +1
    (numpy's own bit unpacking, not the oracle's)."""
    w = np.ascontiguousarray(words, dtype="<u4")
    bits = np.unpackbits(w.view(np.uint8), axis=1, bitorder="little")[:, :r]
    return 2 * bits.astype(np.int64) - 1


def _layer(rng, d_out, d_in, r, s1_bits, s2_bits):
    U = rng.integers(0, 2 ** 32, size=(d_out, r // 32), dtype=np.uint64).astype(np.uint32)
    V = rng.integers(0, 2 ** 32, size=(d_in, r // 32), dtype=np.uint64).astype(np.uint32)
    s1 = np.full(d_out, s1_bits, dtype=np.uint16)
    s2 = np.full(d_in, s2_bits, dtype=np.uint16)
    return (U, V, s1, s2, r)


def _gram(layer):
    U, V, _, _, r = layer
    return _signs(U, r) @ _signs(V, r).T


def _bf16_bits_of_int(v):
    """bf16 bit patterns of integers |v| <= 256 (exact in bf16), via float32."""
    f = np.asarray(v, dtype=np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def _block(seed, d_model=48, d_ff=40, r=32):
    rng = np.random.default_rng(seed)
    gate = _layer(rng, d_ff, d_model, r, F16_ONE, F16_EIGHTH)
    up = _layer(rng, d_ff, d_model, r, F16_ONE, F16_EIGHTH)
    down = _layer(rng, 24, d_ff, r, F16_ONE, F16_ONE)
    x_int = rng.integers(-128, 129, size=(2, d_model))
    return gate, up, down, x_int


@pytest.mark.parametrize("order", ["dense", "factored"])
@pytest.mark.parametrize("seed", [11, 12, 13])
def test_mlp_special_regions_and_unit_scale_down(order, seed):
    gate, up, down, x_int = _block(seed)
    xb = _bf16_bits_of_int(x_int)
    y, S, h = oracle.mlp(gate, up, down, xb, order=order)

    # gate and up exactly: unit s1, s2 = 1/8, integer x
    g = (_gram(gate) @ x_int.T).T / 8.0
    u = (_gram(up) @ x_int.T).T / 8.0
    g16 = oracle.bf16_to_double(oracle.round_bf16(g))
    u16 = oracle.bf16_to_double(oracle.round_bf16(u))
    assert np.mean(g16 != g) > 0.3 and np.mean(u16 != u) > 0.3  # the roundings matter here
    hv = oracle.bf16_to_double(h)

    prod = g16 * u16  # exact: two 8-bit significands
    lo = oracle.round_bf16(prod * (1 - 2.0 ** -40))
    hi = oracle.round_bf16(prod * (1 + 2.0 ** -40))
    big = (g16 >= 40) & (lo == hi)
    assert big.sum() > 10
    np.testing.assert_array_equal(h[big], oracle.round_bf16(prod)[big])
    neg = g16 <= -40
    assert neg.sum() > 10
    assert np.all(np.abs(hv[neg]) <= 1e-15 * np.abs(prod[neg]))
    assert np.all(hv[g16 == 0] == 0)

    # down with unit scales: numpy's matmul of the Gram matrix with h
    Gd = _gram(down).astype(np.float64)
    y_np = hv @ Gd.T
    S_np = np.abs(hv) @ np.abs(Gd).T
    np.testing.assert_allclose(y, y_np, rtol=0, atol=1e-12 * S_np.max())
    np.testing.assert_allclose(S, S_np, rtol=1e-14)


def test_mlp_rows_subset_matches_all_rows():
    gate, up, down, x_int = _block(21)
    xb = _bf16_bits_of_int(x_int)
    y, S, h = oracle.mlp(gate, up, down, xb)
    rows = np.array([0, 5, 23])
    ys, Ss, hs = oracle.mlp(gate, up, down, xb, rows=rows)
    np.testing.assert_array_equal(ys, y[:, rows])
    np.testing.assert_array_equal(Ss, S[:, rows])
    np.testing.assert_array_equal(hs, h)


def test_mlp_zero_gate_gives_zero_block():
    """An all-zero x gives g = u = 0, so h = 0 and the down projection's output is 0."""
    gate, up, down, _ = _block(31)
    xb = np.zeros((1, 48), dtype=np.uint16)
    y, S, h = oracle.mlp(gate, up, down, xb)
    assert np.all(oracle.bf16_to_double(h) == 0) and np.all(y == 0) and np.all(S == 0)


# ----------------------------------------------------------------- planted mistakes
PY_MUTATIONS = [
    # gate and up exchanged in the gated product
    ("h = silu_mul(g16, u16)", "h = silu_mul(u16, g16)"),
    # g not rounded to the bf16 activation dtype
    ("g16 = bf16_to_double(round_bf16(g))", "g16 = g"),
    # u not rounded to the bf16 activation dtype
    ("u16 = bf16_to_double(round_bf16(u))", "u16 = u"),
    # down fed g instead of h
    ("y, S = dense_packed(*down[:4], down[4], h, rows=rows)",
     "y, S = dense_packed(*down[:4], down[4], round_bf16(g16), rows=rows)"),
]


def _run_pins_on_copy(tmp_path, old=None, new=None):
    """Runs the pins above in a subprocess against a copy of the oracle package (CPU only),
    with `old` replaced by `new` in its Python source when given."""
    pkg = tmp_path / "oracle"
    pkg.mkdir()
    src = open(os.path.join(ROOT, "oracle", "__init__.py")).read()
    if old is not None:
        assert old in src, "mutation anchor not found"
        src = src.replace(old, new, 1)
    (pkg / "__init__.py").write_text(src + "\nCOPY_UNDER_TEST = True\n")
    shutil.copy(os.path.join(ROOT, "oracle", "nq_oracle.c"), pkg / "nq_oracle.c")
    env = dict(os.environ, NQ_ORACLE_PKG_DIR=str(tmp_path))
    env.pop("NQ_ORACLE_SO", None)
    return subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                           "-k", "not on_copy", os.path.join(ROOT, "tests", "test_oracle_mlp.py")],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_copy_is_the_one_under_test():
    """Inside the pin subprocess the copy is what `import oracle` finds."""
    if os.environ.get("NQ_ORACLE_PKG_DIR"):
        assert getattr(oracle, "COPY_UNDER_TEST", False)


def test_pins_pass_on_unmodified_on_copy(tmp_path):
    proc = _run_pins_on_copy(tmp_path)
    assert proc.returncode == 0, proc.stdout[-2000:] + proc.stderr[-2000:]


@pytest.mark.parametrize("old,new", PY_MUTATIONS)
def test_pins_fail_on_planted_mistake_on_copy(tmp_path, old, new):
    proc = _run_pins_on_copy(tmp_path, old, new)
    assert proc.returncode != 0, "pins passed on a planted mistake: " + new
