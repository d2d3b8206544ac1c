"""Pins for the CPU oracle (no GPU).

The oracle is checked against things other than itself: hand-worked fixtures, closed
forms, integer matmul from numpy (a library routine) in the special cases that reduce to
it, invariants of the factorisation, and exhaustive enumeration of tiny sign patterns.
Source of the definition: page "NanoQuant: Efficient Sub-1-Bit Quantization of Large
Language Models" (research.samsung.com blog), section 2 "Low-Rank Binary Factorization".
"""
import itertools
import math
import struct

import numpy as np
import pytest

import oracle
from rank_binary_factorized_b200 import synth
from tests.conftest import load_golden


def _hex_words(vals):
    return np.array([int(v, 16) for v in vals], dtype=np.uint32)


def _hex_u16(vals):
    return np.array([int(v, 16) for v in vals], dtype=np.uint16)


def _floats(rows):
    return np.array([[float(v) for v in r] for r in rows], dtype=np.float64)


# --------------------------------------------------------------------------- fixtures
def test_hand_example_dense_signs():
    g = load_golden("hand_example_2x3_r2.txt")
    U = _floats(g["U"]).astype(np.int8)
    V = _floats(g["V"]).astype(np.int8)
    s1 = np.array([float(v) for v in g["s1"]])
    s2 = np.array([float(v) for v in g["s2"]])
    x = _floats(g["x"])
    y, S = oracle.dense_signs(U, V, s1, s2, x)
    np.testing.assert_array_equal(y, _floats(g["y"]))
    np.testing.assert_array_equal(S, _floats(g["S"]))


def test_hand_example_packed_with_cancelling_pad():
    g = load_golden("hand_example_2x3_r2.txt")
    Uw = _hex_words(g["U_words_hex"]).reshape(2, 1)
    Vw = _hex_words(g["V_words_hex"]).reshape(3, 1)
    s1 = _hex_u16(g["s1_f16_hex"])
    s2 = _hex_u16(g["s2_f16_hex"])
    x = np.array([[int(v, 16) for v in row] for row in g["x_bf16_hex"]], dtype=np.uint16)
    np.testing.assert_array_equal(oracle.f16_to_double(s1), [0.5, 2.0])
    np.testing.assert_array_equal(oracle.f16_to_double(s2), [1.0, 0.25, 4.0])
    np.testing.assert_array_equal(oracle.bf16_to_double(x), _floats(g["x"]))
    y, S = oracle.dense_packed(Uw, Vw, s1, s2, 32, x)
    np.testing.assert_array_equal(y, _floats(g["y"]))
    np.testing.assert_array_equal(S, _floats(g["S"]))
    yf = oracle.factored_packed(Uw, Vw, s1, s2, 32, x)
    np.testing.assert_array_equal(yf, _floats(g["y"]))
    # The packed Gram at r = 32 equals the hand-computed rank-2 Gram.
    np.testing.assert_array_equal(oracle.gram_packed(Uw, Vw, 32), [[0, -2, 2], [2, 0, 0]])


def _f32(bits):
    return struct.unpack("<f", struct.pack("<I", bits))[0]


def test_pack_edge_values_golden():
    g = load_golden("pack_edge_values.txt")
    r, ld = int(g["r"][0]), int(g["ld_words"][0])
    L = np.empty((2, r), dtype=np.float32)
    L[0, :11] = [1.0, -1.0, 0.0, -0.0, _f32(1), _f32(0x80000001), _f32(0x7F7FFFFF), _f32(0xFF7FFFFF),
                 np.inf, -np.inf, np.nan]
    for k in range(11, 32):
        L[0, k] = 0.5 if k % 2 else -0.5
    L[0, 32:] = 1.0
    L[1, :] = -1.0
    assert math.copysign(1.0, float(L[0, 3])) < 0  # the -0.0 survived
    P = oracle.pack(L, r=r, ld_words=ld)
    np.testing.assert_array_equal(P[0], _hex_words(g["row0_words_hex"]))
    np.testing.assert_array_equal(P[1], _hex_words(g["row1_words_hex"]))


def test_unpack_bit_order_lsb_first():
    # A single set bit at k gives +1 exactly at element k (word k/32, bit k%32).
    r = 64
    for k in [0, 1, 5, 31, 32, 33, 63]:
        P = np.zeros((1, 2), dtype=np.uint32)
        P[0, k // 32] = np.uint32(1 << (k % 32))
        s = oracle.unpack(P, r)[0]
        expect = -np.ones(r, dtype=np.int8)
        expect[k] = 1
        np.testing.assert_array_equal(s, expect)


def test_pack_unpack_round_trip_and_padding():
    rng = np.random.default_rng(1)
    L = rng.standard_normal((37, 96)).astype(np.float32)
    P = oracle.pack(L, r=96, ld_words=5)
    assert (P[:, 3:] == 0).all()
    S = oracle.unpack(P, 96)
    # A sign times its latent is |latent| for every element: the sign is the latent's sign.
    np.testing.assert_array_equal(S.astype(np.float32) * L, np.abs(L))


# --------------------------------------------------------------------------- formats
def test_f16_decode_known_patterns():
    pats = {0x3C00: 1.0, 0xC000: -2.0, 0x0001: 2.0 ** -24, 0x03FF: 1023 * 2.0 ** -24, 0x0400: 2.0 ** -14,
            0x7BFF: 65504.0, 0x3555: 1365 / 4096, 0x8000: -0.0}
    got = oracle.f16_to_double(np.array(list(pats), dtype=np.uint16))
    np.testing.assert_array_equal(got, list(pats.values()))
    # agrees with numpy's own binary16 on every finite pattern
    allp = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    finite = (allp & 0x7C00) != 0x7C00
    np.testing.assert_array_equal(oracle.f16_to_double(allp[finite]),
                                  allp[finite].view(np.float16).astype(np.float64))


def test_bf16_round_known_values():
    cases = [
        (1.0, 0x3F80),
        (1.0 + 2.0 ** -8, 0x3F80),  # halfway, ties to even (down)
        (1.0 + 3 * 2.0 ** -8, 0x3F82),  # halfway, ties to even (up)
        (1.0 + 2.0 ** -8 + 2.0 ** -40, 0x3F81),  # just above halfway: no double rounding
        (-2.0, 0xC000),
        (1.4621171572600098, 0x3FBB),  # 187/128
        (2.0 ** -133, 0x0001),
        (2.0 ** -134, 0x0000),  # halfway to the smallest subnormal, ties to even
        (3.3895313892515355e38, 0x7F7F),  # largest finite bf16
        (3.3961775292304766e38, 0x7F80),  # rounds up to infinity
    ]
    for v, bits in cases:
        assert int(oracle.round_bf16(np.array([v]))[0]) == bits, (v, hex(bits))
    # bf16 -> fp64 -> bf16 is the identity on finite patterns
    allp = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    finite = (allp & 0x7F80) != 0x7F80
    back = oracle.round_bf16(oracle.bf16_to_double(allp[finite]))
    nonzero = (allp[finite] & 0x7FFF) != 0
    np.testing.assert_array_equal(back[nonzero], allp[finite][nonzero])


def test_silu_mul_values():
    g = np.array([0.0, 1.0, 40.0, -40.0])
    u = np.array([3.0, 2.0, 1.0, 1.0])
    h = oracle.silu_mul(g, u)
    assert int(h[0]) == 0x0000  # silu(0) = 0
    assert int(h[1]) == 0x3FBB  # 2 / (1 + e^-1) = 1.46211... -> 187/128
    assert int(h[2]) == 0x4220  # silu(40) = 40 to within 2^-50 -> bf16(40)
    assert abs(oracle.bf16_to_double(h[3:4])[0]) < 1e-15  # silu(-40) ~ -1.7e-16


# --------------------------------------------------------------------------- Gram
def test_gram_packed_equals_triple_loop_and_integer_matmul():
    rng = synth.rng_for(5, 0)
    d_out, d_in, r = 48, 40, 128
    Uw = synth.sign_words(rng, d_out, r, ld=5)
    Vw = synth.sign_words(rng, d_in, r, ld=4)
    Us = oracle.unpack(Uw, r)
    Vs = oracle.unpack(Vw, r)
    G1 = oracle.gram_packed(Uw, Vw, r)
    G2 = oracle.gram_signs(Us, Vs)
    G3 = Us.astype(np.int64) @ Vs.astype(np.int64).T  # numpy integer matmul
    np.testing.assert_array_equal(G1, G2)
    np.testing.assert_array_equal(G1, G3)
    assert (np.abs(G1) <= r).all() and ((G1 - r) % 2 == 0).all()


def test_brute_force_every_sign_pattern_4x4_r2():
    """All 2^8 x 2^8 pairs (U, V) at d_out = d_in = 4, r = 2.

    The packed path runs at r = 32 with 30 pad columns whose contributions cancel (U pad
    +1; V pad +1 for k = 2..16, -1 for k = 17..31), and must equal the literal triple loop
    and numpy's integer matmul for every pair.
    """
    pats = np.array(list(itertools.product([-1, 1], repeat=8)), dtype=np.int8).reshape(256, 4, 2)

    def to_words(S, pad_u):
        w = np.zeros(S.shape[0], dtype=np.uint32)
        for k in range(2):
            w |= (S[:, k] > 0).astype(np.uint32) << np.uint32(k)
        pad = np.uint32(0xFFFFFFFC) if pad_u else np.uint32(0x0001FFFC)
        return (w | pad).reshape(-1, 1)

    Vall = pats.reshape(1024, 2)  # every V pattern, stacked
    Vw = to_words(Vall, pad_u=False)
    ref_all = None
    for u in range(256):
        U = pats[u]
        G_loop = oracle.gram_signs(U, Vall)  # [4][1024]
        G_mm = U.astype(np.int64) @ Vall.astype(np.int64).T
        G_pk = oracle.gram_packed(to_words(U, pad_u=True), Vw, 32)
        np.testing.assert_array_equal(G_loop, G_mm)
        np.testing.assert_array_equal(G_pk, G_mm)
        ref_all = G_mm if ref_all is None else ref_all
    # forward products on a random sample of the pairs, packed vs literal definition
    rng = np.random.default_rng(11)
    for _ in range(300):
        U, V = pats[rng.integers(256)], pats[rng.integers(256)]
        s1 = np.array([0.5, 2.0, 1.25, -0.75])
        s2 = np.array([1.0, 0.25, 4.0, 0.5])
        xb = synth.f32_to_bf16_bits(rng.standard_normal((3, 4)).astype(np.float32))
        x = oracle.bf16_to_double(xb)
        y1, S1 = oracle.dense_signs(U, V, s1, s2, x)
        s1b = s1.astype(np.float16).view(np.uint16)
        s2b = s2.astype(np.float16).view(np.uint16)
        y2, S2 = oracle.dense_packed(to_words(U, True), to_words(V, False), s1b, s2b, 32, xb)
        np.testing.assert_allclose(y2, y1, rtol=0, atol=1e-13)
        np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-13)


# --------------------------------------------------------------------------- closed forms
def test_unit_scales_reduce_to_integer_matmul():
    """s1 = s2 = 1 and small-integer x: y = (U V^T) x exactly (numpy int64 matmul)."""
    rng = synth.rng_for(6, 0)
    d_out, d_in, r = 33, 70, 96
    Uw = synth.sign_words(rng, d_out, r)
    Vw = synth.sign_words(rng, d_in, r)
    xi = rng.integers(-3, 4, size=(2, d_in))
    ones_o = np.full(d_out, 0x3C00, dtype=np.uint16)
    ones_i = np.full(d_in, 0x3C00, dtype=np.uint16)
    xb = synth.f32_to_bf16_bits(xi.astype(np.float32))
    y, S = oracle.dense_packed(Uw, Vw, ones_o, ones_i, r, xb)
    Us = oracle.unpack(Uw, r).astype(np.int64)
    Vs = oracle.unpack(Vw, r).astype(np.int64)
    G = Us @ Vs.T
    np.testing.assert_array_equal(y, (xi @ G.T).astype(np.float64))
    np.testing.assert_array_equal(S, (np.abs(xi) @ np.abs(G).T).astype(np.float64))
    yf = oracle.factored_packed(Uw, Vw, ones_o, ones_i, r, xb)
    np.testing.assert_array_equal(yf, (xi @ G.T).astype(np.float64))


def test_all_plus_one_closed_form():
    """U = V = all +1: y_i = s1_i * r * sum_j s2_j x_j."""
    rng = synth.rng_for(7, 0)
    d_out, d_in, r = 19, 45, 64
    Uw = np.full((d_out, r // 32), 0xFFFFFFFF, dtype=np.uint32)
    Vw = np.full((d_in, r // 32), 0xFFFFFFFF, dtype=np.uint32)
    s1 = synth.scales_f16(rng, d_out)
    s2 = synth.scales_f16(rng, d_in)
    xb = synth.acts_bf16(rng, (3, d_in))
    s1d, s2d, xd = oracle.f16_to_double(s1), oracle.f16_to_double(s2), oracle.bf16_to_double(xb)
    expect = s1d[None, :] * r * (xd * s2d[None, :]).sum(axis=1, keepdims=True)
    for y in (oracle.dense_packed(Uw, Vw, s1, s2, r, xb)[0], oracle.factored_packed(Uw, Vw, s1, s2, r, xb)):
        np.testing.assert_allclose(y, expect, rtol=1e-13, atol=1e-300)
    # all -1 on one side flips every sign
    y_neg = oracle.dense_packed(np.zeros_like(Uw), Vw, s1, s2, r, xb)[0]
    np.testing.assert_allclose(y_neg, -expect, rtol=1e-13, atol=1e-300)


def test_rank_one_closed_form():
    """r = 1: y = s1 (.) u * (v . (s2 (.) x)); packed r = 32 with all columns equal: 32x that."""
    rng = np.random.default_rng(8)
    d_out, d_in = 23, 31
    u = rng.choice([-1, 1], size=d_out).astype(np.int8)
    v = rng.choice([-1, 1], size=d_in).astype(np.int8)
    s1 = rng.uniform(0.1, 2, d_out)
    s2 = rng.uniform(0.1, 2, d_in)
    x = rng.standard_normal((2, d_in))
    y, _ = oracle.dense_signs(u[:, None], v[:, None], s1, s2, x)
    expect = s1[None, :] * u[None, :] * (x * (s2 * v)[None, :]).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(y, expect, rtol=1e-13)
    # packed: every word is 0 (u = -1) or 0xFFFFFFFF (u = +1)
    Uw = np.where(u > 0, 0xFFFFFFFF, 0).astype(np.uint32)[:, None]
    Vw = np.where(v > 0, 0xFFFFFFFF, 0).astype(np.uint32)[:, None]
    s1b = synth.scales_f16(rng, d_out)
    s2b = synth.scales_f16(rng, d_in)
    xb = synth.acts_bf16(rng, (2, d_in))
    yp, _ = oracle.dense_packed(Uw, Vw, s1b, s2b, 32, xb)
    s1d, s2d, xd = oracle.f16_to_double(s1b), oracle.f16_to_double(s2b), oracle.bf16_to_double(xb)
    expect = 32 * s1d[None, :] * u[None, :] * (xd * (s2d * v)[None, :]).sum(axis=1, keepdims=True)
    np.testing.assert_allclose(yp, expect, rtol=1e-13, atol=1e-300)


def test_associativity_dense_vs_factored():
    layer = synth.make_workload("tiny")[0]
    xb = synth.make_input("tiny", layer.d_in, 3)
    y, S = oracle.dense_packed(layer.U, layer.V, layer.s1, layer.s2, layer.r, xb)
    yf = oracle.factored_packed(layer.U, layer.V, layer.s1, layer.s2, layer.r, xb)
    assert np.max(np.abs(y - yf) / S) < 1e-12
    # a row subset of the dense oracle equals the same rows of the full evaluation
    rows = np.array([0, 7, 255, 128])
    ys, Ss = oracle.dense_packed(layer.U, layer.V, layer.s1, layer.s2, layer.r, xb, rows=rows)
    np.testing.assert_array_equal(ys, y[:, rows])
    np.testing.assert_array_equal(Ss, S[:, rows])


# --------------------------------------------------------------------------- invariants
def test_invariants_of_the_factorisation():
    rng = np.random.default_rng(9)
    d_out, d_in, r = 12, 17, 6
    U = rng.choice([-1, 1], size=(d_out, r)).astype(np.int8)
    V = rng.choice([-1, 1], size=(d_in, r)).astype(np.int8)
    s1 = rng.uniform(0.1, 2, d_out)
    s2 = rng.uniform(0.1, 2, d_in)
    x = rng.standard_normal((2, d_in))
    y, S = oracle.dense_signs(U, V, s1, s2, x)
    # flipping column k of both U and V leaves W unchanged
    F = np.ones(r, dtype=np.int8)
    F[[1, 4]] = -1
    np.testing.assert_allclose(oracle.dense_signs(U * F, V * F, s1, s2, x)[0], y, rtol=1e-14, atol=1e-14)
    # permuting the rank columns leaves W unchanged
    p = rng.permutation(r)
    np.testing.assert_allclose(oracle.dense_signs(U[:, p], V[:, p], s1, s2, x)[0], y, rtol=1e-14, atol=1e-14)
    # negating row i of U negates y_i only
    U2 = U.copy()
    U2[3] *= -1
    y2 = oracle.dense_signs(U2, V, s1, s2, x)[0]
    np.testing.assert_array_equal(y2[:, 3], -y[:, 3])
    np.testing.assert_array_equal(np.delete(y2, 3, axis=1), np.delete(y, 3, axis=1))
    # linear in x; homogeneous in s1 and in s2
    x2 = rng.standard_normal((2, d_in))
    ya = oracle.dense_signs(U, V, s1, s2, x + x2)[0]
    np.testing.assert_allclose(ya, y + oracle.dense_signs(U, V, s1, s2, x2)[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(oracle.dense_signs(U, V, 2 * s1, s2, x)[0], 2 * y)
    np.testing.assert_array_equal(oracle.dense_signs(U, V, s1, 4 * s2, x)[0], 4 * y)
    # s1 indexes output rows, s2 input columns: a one-hot x picks column j of W
    e = np.zeros((1, d_in))
    e[0, 5] = 1.0
    col = oracle.dense_signs(U, V, s1, s2, e)[0][0]
    G = U.astype(np.int64) @ V.astype(np.int64).T
    np.testing.assert_allclose(col, s1 * G[:, 5] * s2[5], rtol=1e-15)
    assert (S >= np.abs(y)).all()


# --------------------------------------------------------------------------- storage
@pytest.mark.parametrize("workload,bpw", [("tiny", 0.75), ("attn7b", 1.0), ("mlp7b", 0.7932),
                                          ("layer70b", 0.5518)])
def test_storage_formula(workload, bpw):
    """r (d_out + d_in) binary values + (d_out + d_in) floats (section 2, after the equation)."""
    bits = weights = scales = 0
    for (_, d_out, d_in, r) in synth.WORKLOADS[workload]:
        bits += r * (d_out + d_in)
        scales += d_out + d_in
        weights += d_out * d_in
    assert round(bits / weights, 4) == bpw
    # the synthetic arrays hold exactly that many sign bits and scale elements
    if workload in ("tiny", "attn7b"):
        projs = synth.make_workload(workload)
        assert sum(32 * (p.U.size + p.V.size) for p in projs) == bits
        assert sum(p.s1.size + p.s2.size for p in projs) == scales
    if workload == "layer70b":
        assert bits // 8 == 59_015_168
