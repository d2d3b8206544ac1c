"""Calibration products on the GPU (nq_lrb_transposed, nq_lrb_scale_grads) against the oracle.

Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models", section 3,
"Phase 3: Scale-Only Model Reconstruction": with U and V frozen, a training step carries the
output gradient back through the layer (its transpose) and needs dL/ds1, dL/ds2.

- transpose: bf16 output held to the forward tolerance 2e-3 * S + 1e-5 + half a bf16 ulp, on
  the decode path (M <= 8) and the tensor cores (M > 8), ragged shapes included;
- scale gradients: fp32 outputs held to 2e-3 * S + 1e-5 + one fp32 rounding, where S is the
  magnitude of the gradient's own terms (the forward's bound weighted by the cotangent).
"""
import numpy as np
import pytest
import torch

import oracle
from rank_binary_factorized_b200 import synth
from tests.gpu_util import (REL, ABS, check_tolerance, download_bf16_bits, need_gpu, nq, upload_bf16,
                            upload_projection)

pytestmark = pytest.mark.gpu


def _acts(seed, B, n):
    return synth.acts_bf16(synth.rng_for(seed, n, B), (B, n))


def _transposed(p, ybar):
    L = upload_projection(p)
    xb = nq().lrb_transposed(L, upload_bf16(ybar))
    nq().sync_status()
    return download_bf16_bits(xb)


def _grads(p, x, ybar):
    L = upload_projection(p)
    g1, g2 = nq().lrb_scale_grads(L, upload_bf16(x), upload_bf16(ybar))
    nq().sync_status()
    return g1.double().cpu().numpy(), g2.double().cpu().numpy()


def _check_grad(g, g_ref, S, what):
    tol = REL * S + ABS + np.abs(g_ref) * 2.0 ** -24
    err = np.abs(g - g_ref)
    bad = err > tol
    assert not bad.any(), "%s: %d of %d outside tolerance, worst err/tol %.3g" % (
        what, int(bad.sum()), bad.size, float(np.max(err / tol)))


@pytest.mark.parametrize("M", [1, 3, 8, 9, 64, 300])
def test_transposed_tiny(M):
    need_gpu()
    p = synth.make_workload("tiny")[0]
    ybar = _acts(950 + M, M, p.d_out)
    xbar = _transposed(p, ybar)
    ref, S = oracle.transposed_packed(p.U, p.V, p.s1, p.s2, p.r, ybar)
    check_tolerance(xbar, ref, S, "transposed tiny M=%d" % M)


@pytest.mark.parametrize("d_out,d_in,r,M", [(77, 1000, 96, 1), (300, 2049, 320, 5), (129, 64, 160, 70),
                                             (640, 200, 2048, 33)])
def test_transposed_ragged(d_out, d_in, r, M):
    need_gpu()
    p = synth.make_projection("ragged-t", d_out, d_in, r, seed=960, key=d_out + d_in)
    ybar = _acts(961, M, d_out)
    xbar = _transposed(p, ybar)
    ref, S = oracle.transposed_packed(p.U, p.V, p.s1, p.s2, p.r, ybar)
    check_tolerance(xbar, ref, S, "transposed ragged %r" % ((d_out, d_in, r, M),))


@pytest.mark.parametrize("workload,M", [("attn7b", 1), ("attn7b", 8), ("prefill70b", 512)])
def test_transposed_full_size_sampled(workload, M):
    need_gpu()
    p = synth.make_workload(workload)[0]
    ybar = _acts(962, M, p.d_out)
    xbar = _transposed(p, ybar)
    cols = np.linspace(0, p.d_in - 1, 48).astype(np.int64)
    ref, S = oracle.transposed_packed(p.U, p.V, p.s1, p.s2, p.r, ybar, cols=cols)
    check_tolerance(xbar[:, cols], ref, S, "transposed %s M=%d" % (workload, M))


@pytest.mark.parametrize("M", [1, 4, 8, 9, 64, 300])
def test_scale_grads_tiny(M):
    need_gpu()
    p = synth.make_workload("tiny")[0]
    x = _acts(970 + M, M, p.d_in)
    ybar = _acts(980 + M, M, p.d_out)
    g1, g2 = _grads(p, x, ybar)
    r1, S1, r2, S2 = oracle.scale_grads_packed(p.U, p.V, p.s1, p.s2, p.r, x, ybar)
    _check_grad(g1, r1, S1, "dL/ds1 tiny M=%d" % M)
    _check_grad(g2, r2, S2, "dL/ds2 tiny M=%d" % M)


@pytest.mark.parametrize("d_out,d_in,r,M", [(77, 1000, 96, 2), (300, 2049, 320, 8), (129, 64, 160, 70),
                                             (1024, 2048, 512, 100)])
def test_scale_grads_ragged(d_out, d_in, r, M):
    need_gpu()
    p = synth.make_projection("ragged-g", d_out, d_in, r, seed=990, key=d_out + d_in)
    x = _acts(991, M, d_in)
    ybar = _acts(992, M, d_out)
    g1, g2 = _grads(p, x, ybar)
    r1, S1, r2, S2 = oracle.scale_grads_packed(p.U, p.V, p.s1, p.s2, p.r, x, ybar)
    _check_grad(g1, r1, S1, "dL/ds1 %r" % ((d_out, d_in, r, M),))
    _check_grad(g2, r2, S2, "dL/ds2 %r" % ((d_out, d_in, r, M),))


def test_scale_grads_repeat_identically_and_share_the_workspace():
    """Two calls give the same bits (fixed summation order), and a forward call on the same
    workspace in between changes nothing."""
    need_gpu()
    p = synth.make_projection("rep", 1024, 2048, 512, seed=993)
    L = upload_projection(p)
    for M in (4, 200):
        x = upload_bf16(_acts(994, M, 2048))
        ybar = upload_bf16(_acts(995, M, 1024))
        ws = torch.zeros(L.workspace_bytes(M), dtype=torch.uint8, device="cuda")
        a1, a2 = nq().lrb_scale_grads(L, x, ybar, ws=ws)
        nq().layer_forward(L, x, ws=ws)
        nq().lrb_transposed(L, ybar, ws=ws)
        b1, b2 = nq().lrb_scale_grads(L, x, ybar, ws=ws)
        nq().sync_status()
        assert torch.equal(a1, b1) and torch.equal(a2, b2)
