"""Pins for the oracle's sign-factor gradients (CPU only).

Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models", section 3,
"Step 3: Factorized Component Refinement": the latent factors are refined through sign()
with straight-through estimators, which need dL/dU and dL/dV of the binary factors.  For
L = sum_b <ybar_b, y_b> the section 2 equation makes L linear in every single entry U_ik
(and V_jk), which fixes the gradient independently of the code under test:

- flipping one sign changes L by exactly -2 U_ik dL/dU_ik (the forward oracle, pinned on
  its own, evaluates both losses);
- sum_k U_ik dL/dU_ik = s1_i dL/ds1_i and sum_k V_jk dL/dV_jk = s2_j dL/ds2_j (the scale
  gradients, pinned on their own);
- unit scales and integer activations reduce both to integer matmuls (numpy);
- the all-+1 closed form.
"""
import numpy as np

import oracle
from rank_binary_factorized_b200 import synth


def _layer(d_out, d_in, r, seed, ld_pad=0):
    return synth.make_projection("sg", d_out, d_in, r, seed=seed, key=d_out + 5 * d_in,
                                 ldu=r // 32 + ld_pad, ldv=r // 32 + ld_pad)


def _acts(seed, B, n):
    return synth.acts_bf16(synth.rng_for(seed, n, B), (B, n))


def _sign(words, row, k):
    return 1 if (int(words[row, k // 32]) >> (k % 32)) & 1 else -1


def _flip(words, row, k):
    w = words.copy()
    w[row, k // 32] ^= np.uint32(1 << (k % 32))
    return w


def _loss(U, V, s1, s2, r, x, ybar):
    y, S = oracle.dense_packed(U, V, s1, s2, r, x)
    yd = oracle.bf16_to_double(ybar)
    return float(np.sum(yd * y)), float(np.sum(np.abs(yd) * S))


def test_flipping_one_sign_changes_the_loss_by_twice_the_gradient():
    p = _layer(40, 72, 64, 1300, ld_pad=1)
    x = _acts(1301, 3, 72)
    ybar = _acts(1302, 3, 40)
    gU, SU, gV, SV = oracle.sign_grads_packed(p.U, p.V, p.s1, p.s2, p.r, x, ybar)
    L0, m0 = _loss(p.U, p.V, p.s1, p.s2, p.r, x, ybar)
    for (i, k) in [(0, 0), (7, 31), (39, 63), (21, 40)]:
        L1, m1 = _loss(_flip(p.U, i, k), p.V, p.s1, p.s2, p.r, x, ybar)
        assert abs((L1 - L0) + 2 * _sign(p.U, i, k) * gU[i, k]) <= 1e-12 * (m0 + m1)
    for (j, k) in [(0, 5), (71, 32), (36, 63)]:
        L1, m1 = _loss(p.U, _flip(p.V, j, k), p.s1, p.s2, p.r, x, ybar)
        assert abs((L1 - L0) + 2 * _sign(p.V, j, k) * gV[j, k]) <= 1e-12 * (m0 + m1)


def test_rank_sums_equal_the_scale_gradients():
    p = _layer(56, 96, 96, 1310)
    x = _acts(1311, 4, 96)
    ybar = _acts(1312, 4, 56)
    gU, SU, gV, SV = oracle.sign_grads_packed(p.U, p.V, p.s1, p.s2, p.r, x, ybar)
    g1, S1, g2, S2 = oracle.scale_grads_packed(p.U, p.V, p.s1, p.s2, p.r, x, ybar)
    su = oracle.unpack(p.U, p.r).astype(np.float64)
    sv = oracle.unpack(p.V, p.r).astype(np.float64)
    s1d, s2d = oracle.f16_to_double(p.s1), oracle.f16_to_double(p.s2)
    np.testing.assert_allclose(np.sum(su * gU, axis=1), s1d * g1, rtol=0, atol=1e-12 * float(SU.sum()))
    np.testing.assert_allclose(np.sum(sv * gV, axis=1), s2d * g2, rtol=0, atol=1e-12 * float(SV.sum()))


def test_unit_scales_reduce_to_integer_matmuls():
    rng = np.random.default_rng(1320)
    d_out, d_in, r, B = 20, 36, 64, 3
    Uw = rng.integers(0, 2 ** 32, size=(d_out, r // 32), dtype=np.uint64).astype(np.uint32)
    Vw = rng.integers(0, 2 ** 32, size=(d_in, r // 32), dtype=np.uint64).astype(np.uint32)
    one_o = np.full(d_out, 0x3C00, dtype=np.uint16)
    one_i = np.full(d_in, 0x3C00, dtype=np.uint16)
    xi = rng.integers(-3, 4, size=(B, d_in))
    yi = rng.integers(-3, 4, size=(B, d_out))
    xb = oracle.round_bf16(xi.astype(np.float64))
    yb = oracle.round_bf16(yi.astype(np.float64))
    Us = oracle.unpack(Uw, r).astype(np.int64)
    Vs = oracle.unpack(Vw, r).astype(np.int64)
    gU, _, gV, _ = oracle.sign_grads_packed(Uw, Vw, one_o, one_i, r, xb, yb)
    np.testing.assert_array_equal(gU, (yi.T @ (xi @ Vs)).astype(np.float64))
    np.testing.assert_array_equal(gV, (xi.T @ (yi @ Us)).astype(np.float64))


def test_all_plus_one_closed_form():
    """U = V = all +1: dL/dU_ik = s1_i sum_b ybar_bi sum_j s2_j x_bj for every k."""
    rng = synth.rng_for(1330, 0)
    d_out, d_in, r = 12, 30, 64
    Uw = np.full((d_out, r // 32), 0xFFFFFFFF, dtype=np.uint32)
    Vw = np.full((d_in, r // 32), 0xFFFFFFFF, dtype=np.uint32)
    s1 = synth.scales_f16(rng, d_out)
    s2 = synth.scales_f16(rng, d_in)
    x = synth.acts_bf16(rng, (2, d_in))
    ybar = synth.acts_bf16(rng, (2, d_out))
    s1d, s2d = oracle.f16_to_double(s1), oracle.f16_to_double(s2)
    xd, yd = oracle.bf16_to_double(x), oracle.bf16_to_double(ybar)
    eU = s1d * np.sum(yd * (xd @ s2d)[:, None], axis=0)
    eV = s2d * np.sum(xd * (yd @ s1d)[:, None], axis=0)
    gU, _, gV, _ = oracle.sign_grads_packed(Uw, Vw, s1, s2, r, x, ybar)
    np.testing.assert_allclose(gU, np.repeat(eU[:, None], r, axis=1), rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(gV, np.repeat(eV[:, None], r, axis=1), rtol=1e-13, atol=1e-300)


def test_selected_entries_and_magnitudes():
    p = _layer(33, 50, 64, 1340, ld_pad=2)
    x = _acts(1341, 2, 50)
    ybar = _acts(1342, 2, 33)
    gU, SU, gV, SV = oracle.sign_grads_packed(p.U, p.V, p.s1, p.s2, p.r, x, ybar)
    ru, rv, ks = np.array([32, 0, 7]), np.array([49, 3]), np.array([63, 0, 31, 32])
    a, Sa, b, Sb = oracle.sign_grads_packed(p.U, p.V, p.s1, p.s2, p.r, x, ybar, rows_u=ru, rows_v=rv, ks=ks)
    np.testing.assert_array_equal(a, gU[np.ix_(ru, ks)])
    np.testing.assert_array_equal(Sa, SU[np.ix_(ru, ks)])
    np.testing.assert_array_equal(b, gV[np.ix_(rv, ks)])
    np.testing.assert_array_equal(Sb, SV[np.ix_(rv, ks)])
    # |dL/dU_ik| never exceeds its magnitude, which does not depend on k (|V_jk| = 1)
    assert np.all(SU >= np.abs(gU)) and np.all(SV >= np.abs(gV))
    np.testing.assert_allclose(SU, np.repeat(SU[:, :1], p.r, axis=1), rtol=1e-14)
