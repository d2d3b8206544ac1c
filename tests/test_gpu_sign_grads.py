"""Sign-factor gradients on the GPU (nq_lrb_sign_grads) against the oracle.

Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models", section 3,
"Step 3: Factorized Component Refinement": the latent factors are refined through sign() with
straight-through estimators, which need dL/dU and dL/dV of the binary factors.  fp32 outputs are
held to 2e-3 * S + 1e-5 + one fp32 rounding, where S is the magnitude of the gradient's own
terms (the forward's bound applied to the expanded sum), on the decode path (M <= 8) and on the
tensor cores (M > 8), ragged shapes and padded output rows included.
"""
import numpy as np
import pytest
import torch

import oracle
from rank_binary_factorized_b200 import synth
from tests.gpu_util import REL, ABS, need_gpu, nq, upload_bf16, upload_projection

pytestmark = pytest.mark.gpu


def _acts(seed, B, n):
    return synth.acts_bf16(synth.rng_for(seed, n, B), (B, n))


def _check(g, g_ref, S, what):
    tol = REL * S + ABS + np.abs(g_ref) * 2.0 ** -24
    err = np.abs(g - g_ref)
    bad = ~(err <= tol)  # NaN counts as bad
    assert not bad.any(), "%s: %d of %d outside tolerance, worst err/tol %.3g" % (
        what, int(bad.sum()), bad.size, float(np.nanmax(err / tol)))


def _run(p, x, ybar, ld_pad=0):
    """GPU gradients as fp64 numpy [rows][r], with ld_pad sentinel columns checked untouched."""
    L = upload_projection(p)
    ld = p.r + ld_pad
    gU = torch.full((p.d_out, ld), -7.0, dtype=torch.float32, device="cuda")
    gV = torch.full((p.d_in, ld), -7.0, dtype=torch.float32, device="cuda")
    nq().lrb_sign_grads(L, upload_bf16(x), upload_bf16(ybar), gU=gU, gV=gV)
    nq().sync_status()
    a, b = gU.double().cpu().numpy(), gV.double().cpu().numpy()
    assert np.all(a[:, p.r:] == -7.0) and np.all(b[:, p.r:] == -7.0)
    return a[:, :p.r], b[:, :p.r]


def _compare(p, x, ybar, what, rows_u=None, rows_v=None, ks=None, ld_pad=0):
    gU, gV = _run(p, x, ybar, ld_pad)
    rU, SU, rV, SV = oracle.sign_grads_packed(p.U, p.V, p.s1, p.s2, p.r, x, ybar, rows_u=rows_u, rows_v=rows_v, ks=ks)
    iu = np.arange(p.d_out) if rows_u is None else np.asarray(rows_u)
    iv = np.arange(p.d_in) if rows_v is None else np.asarray(rows_v)
    kk = np.arange(p.r) if ks is None else np.asarray(ks)
    _check(gU[np.ix_(iu, kk)], rU, SU, what + " dL/dU")
    _check(gV[np.ix_(iv, kk)], rV, SV, what + " dL/dV")
    return gU, gV


@pytest.mark.parametrize("M", [1, 2, 3, 8, 9, 64, 100])
def test_sign_grads_tiny(M):
    need_gpu()
    p = synth.make_workload("tiny")[0]
    _compare(p, _acts(1400 + M, M, p.d_in), _acts(1410 + M, M, p.d_out), "tiny M=%d" % M)


@pytest.mark.parametrize("d_out,d_in,r,M,pad", [(77, 1000, 96, 1, 4), (300, 2049, 320, 5, 0), (129, 64, 160, 70, 4),
                                                 (640, 200, 2048, 33, 8), (40, 72, 32, 200, 0)])
def test_sign_grads_ragged(d_out, d_in, r, M, pad):
    need_gpu()
    p = synth.make_projection("ragged-s", d_out, d_in, r, seed=1420, key=d_out + d_in)
    x = _acts(1421, M, d_in)
    ybar = _acts(1422, M, d_out)
    rng = np.random.default_rng(1423)
    rows_u = np.unique(np.concatenate([[0, d_out - 1], rng.integers(0, d_out, 24)]))
    rows_v = np.unique(np.concatenate([[0, d_in - 1], rng.integers(0, d_in, 24)]))
    ks = np.unique(np.concatenate([[0, r - 1], rng.integers(0, r, 40)]))
    _compare(p, x, ybar, "ragged %r" % ((d_out, d_in, r, M),), rows_u, rows_v, ks, ld_pad=pad)


@pytest.mark.parametrize("workload,M", [("attn7b", 1), ("attn7b", 8), ("prefill70b", 64), ("prefill70b", 2048)])
def test_sign_grads_full_size_sampled(workload, M):
    need_gpu()
    p = synth.make_workload(workload)[0]
    x = _acts(1430, M, p.d_in)
    ybar = _acts(1431, M, p.d_out)
    # decode sizes: three whole rows of each gradient; larger M: a grid of entries
    n = 3 if M <= 8 else (12 if M <= 64 else 3)
    rows_u = np.linspace(0, p.d_out - 1, n).astype(np.int64)
    rows_v = np.linspace(0, p.d_in - 1, n).astype(np.int64)
    ks = None if M <= 8 else np.linspace(0, p.r - 1, n).astype(np.int64)
    gU, gV = _compare(p, x, ybar, "%s M=%d" % (workload, M), rows_u, rows_v, ks)
    assert np.all(np.isfinite(gU)) and np.all(np.isfinite(gV))


def test_sign_grads_repeat_identically():
    need_gpu()
    p = synth.make_projection("rep-s", 1024, 2048, 512, seed=1460)
    L = upload_projection(p)
    for M in (4, 200):
        x = upload_bf16(_acts(1461, M, 2048))
        ybar = upload_bf16(_acts(1462, M, 1024))
        a = nq().lrb_sign_grads(L, x, ybar)
        b = nq().lrb_sign_grads(L, x, ybar)
        nq().sync_status()
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
