"""Prefill path (nq_lrb_matmul, tcgen05 tensor cores) against the CPU oracle.

- floating parity at the stated tolerance on ragged shapes (d_out, r, d_in and M not
  multiples of the 128 x 64 x 256 tiles) and on the 70B gate projection at M = 64, 512,
  2048 (sampled outputs, the launch the benchmark times);
- integer-exact regime: s1 = s2 = 1, x in {-1, 0, 1} and |t| <= 2048, where every fp16
  operand and intermediate is an exact integer, so the GPU must equal bf16(y_ref) bitwise;
- every 4 x 2 sign pattern (stacked, r = 32 with cancelling pad columns), bitwise.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
from rank_binary_factorized_b200 import synth
from tests.gpu_util import (ABS, REL, bf16_bits_to_f64, check_tolerance, download_bf16_bits, half_ulp_bf16, need_gpu, nq,
                            upload_bf16, upload_projection)

pytestmark = pytest.mark.gpu


def gpu_matmul(p, xb, fn="lrb_matmul", ld_align_words=4):
    L = upload_projection(p, ld_align_words=ld_align_words)
    y = getattr(nq(), fn)(L, upload_bf16(xb))
    nq().sync_status()
    return download_bf16_bits(y)


@pytest.mark.parametrize("M", [9, 16, 64, 100, 256, 300])
def test_tiny_layer_token_counts(M):
    need_gpu()
    p = synth.make_workload("tiny")[0]
    xb = synth.make_input("tiny", p.d_in, M, key=100 + M)
    y = gpu_matmul(p, xb)
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
    check_tolerance(y, y_ref, S, "prefill tiny M=%d" % M)


@pytest.mark.parametrize("d_out,d_in,r,ldu,ldv,M", [
    (77, 1000, 96, 3, 3, 20),
    (300, 2049, 320, 10, 11, 70),
    (129, 64, 160, 5, 8, 257),
    (1, 8, 32, 1, 1, 9),
    (640, 200, 2048, 64, 66, 33),
])
@pytest.mark.parametrize("align", [1, 4])
def test_ragged_and_padded(d_out, d_in, r, ldu, ldv, M, align):
    # align 1 keeps the given row strides (odd ones load the packed signs with plain loads);
    # align 4 pads them to 16 bytes (the signs arrive by TMA)
    need_gpu()
    p = synth.make_projection("ragged", d_out, d_in, r, seed=402, key=d_out + 3 * d_in, ldu=ldu, ldv=ldv)
    xb = synth.acts_bf16(synth.rng_for(403, d_in, M), (M, d_in))
    y = gpu_matmul(p, xb, ld_align_words=align)
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
    check_tolerance(y, y_ref, S, "prefill ragged %r align %d" % ((d_out, d_in, r, ldu, ldv, M), align))


@pytest.mark.parametrize("d_out,d_in,r,M", [(256, 512, 128, 64), (1024, 2048, 512, 300), (4096, 1024, 1024, 40)])
def test_integer_exact_bitwise(d_out, d_in, r, M):
    need_gpu()
    p = synth.make_projection("int", d_out, d_in, r, seed=404, key=d_out + M)
    p.s1 = np.full(d_out, 0x3C00, dtype=np.uint16)
    p.s2 = np.full(d_in, 0x3C00, dtype=np.uint16)
    xi = synth.rng_for(405, d_out, M).integers(-1, 2, size=(M, d_in)).astype(np.float32)
    xb = synth.f32_to_bf16_bits(xi)
    y = gpu_matmul(p, xb)
    rows = np.arange(d_out) if d_out <= 1024 else np.linspace(0, d_out - 1, 300).astype(np.int64)
    y_ref, _ = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb, rows=rows)
    np.testing.assert_array_equal(y[:, rows], oracle.round_bf16(y_ref))


def test_every_sign_pattern_4x2_bitwise():
    need_gpu()
    pats = np.array(list(itertools.product([-1, 1], repeat=8)), dtype=np.int8).reshape(256 * 4, 2)

    def words(S, pad):
        w = np.zeros(S.shape[0], dtype=np.uint32)
        for k in range(2):
            w |= (S[:, k] > 0).astype(np.uint32) << np.uint32(k)
        return (w | np.uint32(pad)).reshape(-1, 1)

    p = synth.Projection("patterns", 1024, 1024, 32, words(pats, 0xFFFFFFFC), words(pats, 0x0001FFFC),
                         np.full(1024, 0x3C00, dtype=np.uint16), np.full(1024, 0x3C00, dtype=np.uint16))
    xi = synth.rng_for(406).integers(-1, 2, size=(24, 1024)).astype(np.float32)
    xb = synth.f32_to_bf16_bits(xi)
    y = gpu_matmul(p, xb)
    y_ref, _ = oracle.dense_packed(p.U, p.V, p.s1, p.s2, 32, xb)
    np.testing.assert_array_equal(y, oracle.round_bf16(y_ref))


@pytest.mark.parametrize("M", [64, 512, 2048])
def test_full_size_70b_gate_sampled(M):
    """The 70B gate projection (28672 x 8192, r = 3520) at the benchmark's token counts;
    sampled output features for every token."""
    need_gpu()
    p = synth.make_workload("prefill70b")[0]
    xb = synth.make_input("prefill70b", p.d_in, M, key=M)
    y = gpu_matmul(p, xb)
    # rows of the last weight tiles too
    tail = [p.d_out - 512, p.d_out - 300, p.d_out - 129, p.d_out - 128, p.d_out - 1]
    rows = np.unique(np.concatenate([[0, 127, 128], tail, np.linspace(0, p.d_out - 1, 40).astype(np.int64)]))
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb, rows=rows)
    check_tolerance(y[:, rows], y_ref, S, "prefill 70B gate M=%d" % M)



def test_layer_forward_dispatches_to_matmul_and_is_deterministic():
    need_gpu()
    p = synth.make_workload("tiny")[0]
    xb = synth.make_input("tiny", p.d_in, 33, key=7)
    y1 = gpu_matmul(p, xb, fn="layer_forward")
    y2 = gpu_matmul(p, xb, fn="lrb_matmul")
    np.testing.assert_array_equal(y1, y2)


def test_matmul_small_m_matches_matvec_tolerance():
    """nq_lrb_matmul accepts M <= 8 too (the tensor-core path with a 16-token tile)."""
    need_gpu()
    p = synth.make_workload("tiny")[0]
    xb = synth.make_input("tiny", p.d_in, 3, key=8)
    y = gpu_matmul(p, xb)
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
    check_tolerance(y, y_ref, S, "prefill M=3")


def test_one_workspace_shared_by_decode_and_prefill():
    """Decode and prefill calls of different shapes share one zero-initialised workspace."""
    need_gpu()
    p = synth.make_projection("shared", 640, 1536, 256, seed=407, key=1)
    L = upload_projection(p)
    need = max(L.workspace_bytes(M) for M in (1, 8, 300))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    outs = []
    for M in (1, 300, 8, 77, 3, 300, 1):
        xb = synth.acts_bf16(synth.rng_for(408, M), (M, p.d_in))
        y = nq().layer_forward(L, upload_bf16(xb), ws=ws)
        outs.append((xb, y))
    nq().sync_status()
    for xb, y in outs:
        y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
        check_tolerance(download_bf16_bits(y), y_ref, S, "shared workspace M=%d" % xb.shape[0])


def _rows_scaled(xb, exps):
    """bf16 rows multiplied by 2^e (exact; e = None gives an all-zero row)."""
    xf = (np.asarray(xb, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for m, e in enumerate(exps):
        xf[m] = 0.0 if e is None else np.ldexp(xf[m], e)
    return oracle.round_bf16(xf)


@pytest.mark.parametrize("d_out,d_in,r", [(300, 2048, 256), (129, 1000, 96)])
def test_rows_beyond_and_below_fp16_range(d_out, d_in, r):
    """Each row gets its own power of two before the fp16 conversion: rows scaled by 2^-120 up to
    2^124 (|x s2| far above 65504, sums of |x s2| beyond fp32's range, and values far below fp16's
    smallest normal) and an all-zero row, in one call, each within its own tolerance and finite;
    the zero row is zero."""
    need_gpu()
    p = synth.make_projection("range", d_out, d_in, r, seed=2400, key=d_out)
    exps = [-120, -30, 0, 20, 80, None, 40, -60, 124, 10]  # M = 10 > 8: the tensor-core path
    xb = _rows_scaled(synth.acts_bf16(synth.rng_for(2401, d_in), (len(exps), d_in)), exps)
    y = gpu_matmul(p, xb)
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
    assert np.all(np.isfinite(y_ref))
    got = bf16_bits_to_f64(y)
    assert np.all(np.isfinite(got))
    for m, e in enumerate(exps):
        if e is None:
            assert np.all(y[m] & 0x7FFF == 0)
            continue
        # row m is a base row times 2^e, so is everything it produces: the absolute part of the
        # bound scales with it (else it would hide any error of a tiny row)
        tol = REL * S[m] + ABS * 2.0 ** e + half_ulp_bf16(y_ref[m])
        err = np.abs(got[m] - y_ref[m])
        assert np.all(err <= tol), "row 2^%d: max err/tol %.3g" % (e, float((err / tol).max()))


def test_intermediate_beyond_fp16_range():
    """Unit scales and |x| around 1000: every z fits fp16 but the sums t over 8192 rows reach
    about 10^5, beyond 65504; the per-row power of two keeps t in range."""
    need_gpu()
    d_out, d_in, r, M = 512, 8192, 256, 12
    p = synth.make_projection("trange", d_out, d_in, r, seed=2402)
    p.s1 = np.full(d_out, 0x3C00, dtype=np.uint16)
    p.s2 = np.full(d_in, 0x3C00, dtype=np.uint16)
    xb = _rows_scaled(synth.acts_bf16(synth.rng_for(2403, d_in), (M, d_in)), [10] * M)
    # the premise, by numpy alone: t = V^T x with V's unpacked signs (unit s2)
    vbits = np.unpackbits(np.ascontiguousarray(p.V, dtype="<u4").view(np.uint8), axis=1, bitorder="little")[:, :r]
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    t = xf @ (2.0 * vbits - 1.0)
    assert np.abs(xf).max() < 65504 and np.abs(t).max() > 65504
    y = gpu_matmul(p, xb)
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
    check_tolerance(y, y_ref, S, "prefill |t| > 65504")


def test_scale_grads_prefill_rows_beyond_fp16_range():
    """The scale gradients' tensor-core path sums over rows in fp64 after undoing each row's
    power of two: rows at 2^40 and 2^-40 in one call match the oracle's gradients."""
    need_gpu()
    d_out, d_in, r = 200, 512, 128
    p = synth.make_projection("gscale", d_out, d_in, r, seed=2404)
    exps = [40, 0, -40, 10, 0, -10, 20, 0, 5, -5]
    xb = _rows_scaled(synth.acts_bf16(synth.rng_for(2405, d_in), (len(exps), d_in)), exps)
    yb = synth.acts_bf16(synth.rng_for(2406, d_out), (len(exps), d_out))
    L = upload_projection(p)
    g1, g2 = nq().lrb_scale_grads(L, upload_bf16(xb), upload_bf16(yb))
    nq().sync_status()
    ref1, S1, ref2, S2 = oracle.scale_grads_packed(p.U, p.V, p.s1, p.s2, p.r, xb, yb)
    g1 = g1.cpu().numpy().astype(np.float64)
    g2 = g2.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(g1)) and np.all(np.isfinite(g2))
    # fp32 outputs: the stated bound plus the output rounding (2^-24 relative)
    assert np.all(np.abs(g1 - ref1) <= 2e-3 * S1 + 1e-5 + 2.0 ** -24 * np.abs(ref1))
    assert np.all(np.abs(g2 - ref2) <= 2e-3 * S2 + 1e-5 + 2.0 ** -24 * np.abs(ref2))
