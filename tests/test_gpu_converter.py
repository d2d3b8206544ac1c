"""nq_lrb_from_latent on the GPU against the oracle's converter.

Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models", section 3,
"Magnitude Balancing and Scale Extraction" and "Phase 3" packing.  The packed signs must be
bit-identical.  eta and the fp64 scales are sums of the same fp32 values in another order,
so they agree to fp64 rounding.  The fp16 scales are a rounding decision taken on those fp64
values: they must be identical too, except where the oracle's value lies within 1e-12
(relative) of an fp16 rounding midpoint.  There the order of the fp64 sums may legitimately
decide the rounding; the test checks that no mismatch falls elsewhere.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_util import need_gpu, nq

pytestmark = pytest.mark.gpu


def _near_f16_midpoint(v):
    """True where v is within 1e-12 (relative) of the midpoint of two adjacent fp16 values."""
    lo = oracle.f16_to_double(oracle.double_to_f16(v))
    step = np.maximum(np.abs(lo) * 2.0 ** -10, 2.0 ** -24)
    mid_up, mid_dn = lo + step / 2, lo - step / 2
    tol = 1e-12 * np.maximum(np.abs(v), 2.0 ** -24)
    return (np.abs(v - mid_up) <= tol) | (np.abs(v - mid_dn) <= tol)


def _run(Uh, Vh, ld_align=4):
    L, eta = nq().lrb_from_latent(torch.from_numpy(Uh).cuda(), torch.from_numpy(Vh).cuda(), ld_align_words=ld_align)
    nq().sync_status()
    return (L.U.cpu().numpy().view(np.uint32), L.V.cpu().numpy().view(np.uint32),
            L.s1.cpu().numpy().view(np.uint16), L.s2.cpu().numpy().view(np.uint16), float(eta.item()))


@pytest.mark.parametrize("d_out,d_in,r,su,sv,align", [
    (256, 512, 128, 1.0, 1.0, 4),
    (77, 130, 96, 5.0, 0.01, 1),
    (1, 33, 32, 1e-3, 1.0, 4),
    (4096, 4096, 2048, 0.3, 2.0, 4),
    (28672, 8192, 3520, 0.05, 0.02, 4),
])
def test_from_latent_matches_the_oracle(d_out, d_in, r, su, sv, align):
    need_gpu()
    rng = np.random.default_rng(d_out + 3 * d_in + r)
    Uh = (su * rng.standard_normal((d_out, r))).astype(np.float32)
    Vh = (sv * rng.standard_normal((d_in, r))).astype(np.float32)
    Uh[0, :3] = [0.0, -0.0, np.nan]
    U, V, s1, s2, eta = _run(Uh, Vh, align)
    ldu, ldv = U.shape[1], V.shape[1]
    Ur, Vr, s1r, s2r, eta_r, s1d, s2d = oracle.from_latent(Uh, Vh, ldu=ldu, ldv=ldv)
    np.testing.assert_array_equal(U, Ur)
    np.testing.assert_array_equal(V, Vr)
    assert abs(eta - eta_r) <= 1e-12 * eta_r
    for got, want, vd, name in ((s1, s1r, s1d, "s1"), (s2, s2r, s2d, "s2")):
        bad = got != want
        assert not np.any(bad & ~_near_f16_midpoint(vd)), "%s: %d fp16 mismatches away from rounding midpoints" % (
            name, int(np.sum(bad & ~_near_f16_midpoint(vd))))


def test_from_latent_zero_factor_and_layer_use():
    """A zero latent gives eta = 1 and zero scales; the returned Layer runs the forward path."""
    need_gpu()
    rng = np.random.default_rng(7)
    Uh = np.zeros((64, 64), dtype=np.float32)
    Vh = rng.standard_normal((96, 64)).astype(np.float32)
    U, V, s1, s2, eta = _run(Uh, Vh)
    assert eta == 1.0 and np.all(s1 == 0) and np.all(U[:, :2] == 0xFFFFFFFF)
    L, _ = nq().lrb_from_latent(torch.from_numpy(rng.standard_normal((64, 64)).astype(np.float32)).cuda(),
                                torch.from_numpy(Vh).cuda())
    y = nq().layer_forward(L, torch.zeros((1, 96), dtype=torch.bfloat16, device="cuda").normal_())
    nq().sync_status()
    assert torch.isfinite(y.float()).all()
