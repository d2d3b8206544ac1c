"""Pins for the oracle's latent-to-layer converter and its fp16 encoder (CPU only).

Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models", section 3,
"Magnitude Balancing and Scale Extraction": eta = sqrt(||Vh||_F / ||Uh||_F), U := eta Uh,
V := Vh / eta, s1 and s2 the mean absolute values of the rows of U and V.  "Phase 3" then
packs sign(U), sign(V).  Pinned by the binary16 format itself and by closed forms and
invariances of the balancing, each independent of the code under test.
"""
import numpy as np

import oracle


def _finite_f16_patterns():
    p = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    return p[((p >> 10) & 0x1F) != 0x1F]


def test_f16_encoder_round_trips_every_finite_pattern():
    p = _finite_f16_patterns()
    back = oracle.double_to_f16(oracle.f16_to_double(p))
    np.testing.assert_array_equal(back, p)  # +0 and -0 included


def test_f16_encoder_rounds_midpoints_to_even():
    pos = np.arange(0, 0x7BFF, dtype=np.uint16)  # adjacent finite non-negative pairs (p, p + 1)
    lo = oracle.f16_to_double(pos)
    hi = oracle.f16_to_double(pos + 1)
    mid = (lo + hi) / 2.0  # exact in fp64
    got = oracle.double_to_f16(mid)
    want = np.where(pos % 2 == 0, pos, pos + 1).astype(np.uint16)
    np.testing.assert_array_equal(got, want)
    # just below / above a midpoint goes down / up
    np.testing.assert_array_equal(oracle.double_to_f16(np.nextafter(mid, 0)), pos)
    np.testing.assert_array_equal(oracle.double_to_f16(np.nextafter(mid, np.inf)), (pos + 1).astype(np.uint16))
    # overflow: the midpoint of 65504 and 65536 rounds to even, i.e. to infinity
    assert oracle.double_to_f16(65519.999) == 0x7BFF and oracle.double_to_f16(65520.0) == 0x7C00


def _latents(seed, d_out, d_in, r, su=1.0, sv=1.0):
    rng = np.random.default_rng(seed)
    return ((su * rng.standard_normal((d_out, r))).astype(np.float32),
            (sv * rng.standard_normal((d_in, r))).astype(np.float32))


def test_balanced_norms_meet_at_the_geometric_mean():
    Uh, Vh = _latents(1200, 40, 72, 64, su=3.0, sv=0.2)
    U, V, s1, s2, eta, s1d, s2d = oracle.from_latent(Uh, Vh)
    nu, nv = np.linalg.norm(Uh.astype(np.float64)), np.linalg.norm(Vh.astype(np.float64))
    assert abs(eta - np.sqrt(nv / nu)) <= 1e-14 * eta
    a = np.linalg.norm(eta * Uh.astype(np.float64))
    b = np.linalg.norm(Vh.astype(np.float64) / eta)
    g = np.sqrt(nu * nv)
    assert abs(a - g) <= 1e-12 * g and abs(b - g) <= 1e-12 * g


def test_scales_are_row_mean_absolute_values():
    d_out, d_in, r = 6, 5, 32
    c = np.array([1.0, -2.0, 0.5, 0.0, -0.25, 3.0], dtype=np.float32)
    Uh = np.repeat(c[:, None], r, axis=1)
    Vh = np.repeat(np.array([2.0, -1.0, 4.0, -0.5, 1.0], dtype=np.float32)[:, None], r, axis=1)
    U, V, s1, s2, eta, s1d, s2d = oracle.from_latent(Uh, Vh)
    np.testing.assert_allclose(s1d, eta * np.abs(c.astype(np.float64)), rtol=1e-15)
    np.testing.assert_allclose(s2d, np.abs(Vh[:, 0].astype(np.float64)) / eta, rtol=1e-15)
    np.testing.assert_array_equal(s1, oracle.double_to_f16(s1d))
    np.testing.assert_array_equal(s2, oracle.double_to_f16(s2d))


def test_exchanging_the_factors_inverts_eta_and_swaps_the_scales():
    Uh, Vh = _latents(1201, 30, 50, 64, su=2.0)
    _, _, _, _, eta, s1d, s2d = oracle.from_latent(Uh, Vh)
    _, _, _, _, eta_x, s1x, s2x = oracle.from_latent(Vh, Uh)
    assert abs(eta * eta_x - 1.0) <= 1e-14
    np.testing.assert_allclose(s1x, s2d, rtol=1e-13)
    np.testing.assert_allclose(s2x, s1d, rtol=1e-13)


def test_scaling_a_factor_scales_the_reconstruction():
    """Uh -> a Uh multiplies U Vh^T by a; the balanced scales split it evenly: every
    s1_i s2_j is multiplied by a, and the signs do not change."""
    Uh, Vh = _latents(1202, 24, 40, 64)
    a = 4.0  # a power of two: a * Uh is exact in fp32
    U, V, _, _, eta, s1d, s2d = oracle.from_latent(Uh, Vh)
    Ua, Va, _, _, eta_a, s1a, s2a = oracle.from_latent(a * Uh, Vh)
    np.testing.assert_array_equal(Ua, U)
    np.testing.assert_array_equal(Va, V)
    assert abs(eta_a * np.sqrt(a) - eta) <= 1e-14 * eta
    np.testing.assert_allclose(np.outer(s1a, s2a), a * np.outer(s1d, s2d), rtol=1e-13)


def test_signs_are_the_pack_of_the_latents_and_zero_latents_stay_neutral():
    Uh, Vh = _latents(1203, 20, 33, 96)
    Uh[0, :5] = 0.0
    Uh[1, 3] = -0.0
    U, V, *_ = oracle.from_latent(Uh, Vh, ldu=4, ldv=5)
    np.testing.assert_array_equal(U, oracle.pack(Uh, 96, ld_words=4))
    np.testing.assert_array_equal(V, oracle.pack(Vh, 96, ld_words=5))
    Z = np.zeros((8, 32), dtype=np.float32)
    Uz, Vz, s1, s2, eta, s1d, s2d = oracle.from_latent(Z, Vh[:, :32])
    assert eta == 1.0 and np.all(s1 == 0) and np.all(Uz == 0xFFFFFFFF)
