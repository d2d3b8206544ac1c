"""Pins for the oracle's calibration products (CPU only).

Phase 3 of the method ("Scale-Only Model Reconstruction", page "NanoQuant: Efficient
Sub-1-Bit Quantization of Large Language Models", section 3) freezes U and V and optimises s1
and s2.  Its training step needs the layer's transpose and the derivatives of the output with
respect to both scale vectors.  Each is pinned here by mathematics, independently of the code
under test:

- the adjoint identity <ybar, W x> = <W^T ybar, x>;
- the transpose of a layer equals the forward of the layer with (U, s1) and (V, s2) exchanged;
- the all-+1 closed form;
- integer matmuls at unit scales;
- L = sum <ybar, y> is linear in every scale entry.  So Euler's identity
  sum_i s1_i dL/ds1_i = L = sum_j s2_j dL/ds2_j holds, and a finite difference is exact.
"""
import numpy as np

import oracle
from rank_binary_factorized_b200 import synth


def _layer(d_out, d_in, r, seed, ld_pad=0):
    p = synth.make_projection("cal", d_out, d_in, r, seed=seed, key=d_out + 7 * d_in,
                              ldu=r // 32 + ld_pad, ldv=r // 32 + ld_pad)
    return p


def _acts(seed, B, n):
    return synth.acts_bf16(synth.rng_for(seed, n, B), (B, n))


def test_transpose_adjoint_identity():
    for (d_out, d_in, r, pad) in [(256, 512, 128, 0), (77, 130, 96, 1)]:
        p = _layer(d_out, d_in, r, 900, pad)
        x = _acts(901, 3, d_in)
        ybar = _acts(902, 3, d_out)
        y, Sy = oracle.dense_packed(p.U, p.V, p.s1, p.s2, r, x)
        xbar, Sx = oracle.transposed_packed(p.U, p.V, p.s1, p.s2, r, ybar)
        xd, yd = oracle.bf16_to_double(x), oracle.bf16_to_double(ybar)
        lhs = float(np.sum(yd * y))
        rhs = float(np.sum(xbar * xd))
        scale = float(np.sum(np.abs(yd) * Sy))
        assert abs(lhs - rhs) <= 1e-12 * scale


def test_transpose_is_forward_of_exchanged_layer():
    p = _layer(77, 130, 96, 903, 1)
    ybar = _acts(904, 2, 77)
    xbar, S = oracle.transposed_packed(p.U, p.V, p.s1, p.s2, p.r, ybar)
    y2, S2 = oracle.dense_packed(p.V, p.U, p.s2, p.s1, p.r, ybar)
    np.testing.assert_array_equal(xbar, y2)
    np.testing.assert_array_equal(S, S2)
    cols = np.array([0, 129, 64, 3])
    xs, Ss = oracle.transposed_packed(p.U, p.V, p.s1, p.s2, p.r, ybar, cols=cols)
    np.testing.assert_array_equal(xs, xbar[:, cols])
    np.testing.assert_array_equal(Ss, S[:, cols])


def test_transpose_all_plus_one_closed_form():
    """U = V = all +1: xbar_j = s2_j * r * sum_i s1_i ybar_i."""
    rng = synth.rng_for(905, 0)
    d_out, d_in, r = 21, 40, 64
    Uw = np.full((d_out, r // 32), 0xFFFFFFFF, dtype=np.uint32)
    Vw = np.full((d_in, r // 32), 0xFFFFFFFF, dtype=np.uint32)
    s1 = synth.scales_f16(rng, d_out)
    s2 = synth.scales_f16(rng, d_in)
    ybar = synth.acts_bf16(rng, (2, d_out))
    s1d, s2d, yd = oracle.f16_to_double(s1), oracle.f16_to_double(s2), oracle.bf16_to_double(ybar)
    expect = s2d[None, :] * r * (yd * s1d[None, :]).sum(axis=1, keepdims=True)
    xbar, _ = oracle.transposed_packed(Uw, Vw, s1, s2, r, ybar)
    np.testing.assert_allclose(xbar, expect, rtol=1e-13, atol=1e-300)


def test_unit_scales_reduce_to_integer_matmuls():
    """s1 = s2 = 1 and integer activations: the transpose is ybar G and the scale gradients
    are row sums of ybar (.) (x G^T) and of x (.) (ybar G), all exact integers."""
    rng = np.random.default_rng(906)
    d_out, d_in, r, B = 24, 33, 64, 3
    Uw = rng.integers(0, 2 ** 32, size=(d_out, r // 32), dtype=np.uint64).astype(np.uint32)
    Vw = rng.integers(0, 2 ** 32, size=(d_in, r // 32), dtype=np.uint64).astype(np.uint32)
    one_o = np.full(d_out, 0x3C00, dtype=np.uint16)
    one_i = np.full(d_in, 0x3C00, dtype=np.uint16)
    xi = rng.integers(-3, 4, size=(B, d_in))
    yi = rng.integers(-3, 4, size=(B, d_out))
    xb = oracle.round_bf16(xi.astype(np.float64))
    yb = oracle.round_bf16(yi.astype(np.float64))
    G = oracle.unpack(Uw, r).astype(np.int64) @ oracle.unpack(Vw, r).astype(np.int64).T
    xbar, _ = oracle.transposed_packed(Uw, Vw, one_o, one_i, r, yb)
    np.testing.assert_array_equal(xbar, (yi @ G).astype(np.float64))
    g1, _, g2, _ = oracle.scale_grads_packed(Uw, Vw, one_o, one_i, r, xb, yb)
    np.testing.assert_array_equal(g1, (yi * (xi @ G.T)).sum(axis=0).astype(np.float64))
    np.testing.assert_array_equal(g2, (xi * (yi @ G)).sum(axis=0).astype(np.float64))


def test_scale_grads_euler_identity():
    p = _layer(96, 160, 64, 907)
    x = _acts(908, 4, 160)
    ybar = _acts(909, 4, 96)
    y, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, x)
    g1, S1, g2, S2 = oracle.scale_grads_packed(p.U, p.V, p.s1, p.s2, p.r, x, ybar)
    L = float(np.sum(oracle.bf16_to_double(ybar) * y))
    s1d, s2d = oracle.f16_to_double(p.s1), oracle.f16_to_double(p.s2)
    bound = 1e-12 * float(np.sum(s1d * S1))
    assert abs(float(np.sum(s1d * g1)) - L) <= bound
    assert abs(float(np.sum(s2d * g2)) - L) <= bound
    # the magnitudes are those of the same terms
    assert np.all(S1 >= np.abs(g1)) and np.all(S2 >= np.abs(g2))


def test_scale_grads_finite_difference_is_exact():
    """L is linear in s1_i (and in s2_j): changing one scale by d changes L by d * grad."""
    p = _layer(40, 72, 64, 910)
    x = _acts(911, 2, 72)
    ybar = _acts(912, 2, 40)
    yd = oracle.bf16_to_double(ybar)
    g1, S1, g2, S2 = oracle.scale_grads_packed(p.U, p.V, p.s1, p.s2, p.r, x, ybar)

    def loss(s1, s2):
        y, S = oracle.dense_packed(p.U, p.V, s1, s2, p.r, x)
        return float(np.sum(yd * y)), float(np.sum(np.abs(yd) * S))

    L0, mag = loss(p.s1, p.s2)
    for i in (0, 17, 39):
        s1 = p.s1.copy()
        s1[i] = 0x3A00  # fp16 0.75
        d = 0.75 - float(oracle.f16_to_double(p.s1[i:i + 1])[0])
        L1, mag1 = loss(s1, p.s2)
        assert abs((L1 - L0) - d * g1[i]) <= 1e-12 * (mag + mag1 + abs(d) * S1[i])
    for j in (0, 31, 71):
        s2 = p.s2.copy()
        s2[j] = 0xB800  # fp16 -0.5
        d = -0.5 - float(oracle.f16_to_double(p.s2[j:j + 1])[0])
        L1, mag1 = loss(p.s1, s2)
        assert abs((L1 - L0) - d * g2[j]) <= 1e-12 * (mag + mag1 + abs(d) * S2[j])
