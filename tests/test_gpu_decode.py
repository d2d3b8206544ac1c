"""Decode path (nq_lrb_matvec, M = 1..8) against the CPU oracle.

- floating parity: |y - y_ref| <= 2e-3 * S + 1e-5 per output (S = sum_j |W_ij x_j|);
- integer-exact regime (s1 = s2 = 1, x in {-1, 0, 1}): every fp32 intermediate is exact,
  so the GPU output must equal bf16(y_ref) bit for bit;
- every sign pattern of 4 x 2 factors (packed at r = 32 with cancelling pad columns);
- full-size Llama-2 projections on sampled output rows;
- ragged sizes, padded leading dimensions, run-to-run determinism.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
from rank_binary_factorized_b200 import synth
from tests.gpu_util import (bf16_bits_to_f64, check_tolerance, download_bf16_bits, need_gpu, nq, upload_bf16,
                            upload_projection)

pytestmark = pytest.mark.gpu


def gpu_forward(p, xb, fn="lrb_matvec", ld_align_words=4):
    L = upload_projection(p, ld_align_words=ld_align_words)
    x = upload_bf16(xb)
    y = getattr(nq(), fn)(L, x)
    nq().sync_status()
    return download_bf16_bits(y)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8])
def test_tiny_all_batches(M):
    need_gpu()
    p = synth.make_workload("tiny")[0]
    xb = synth.make_input("tiny", p.d_in, M)
    y = gpu_forward(p, xb)
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
    check_tolerance(y, y_ref, S, "tiny M=%d" % M)


@pytest.mark.parametrize("d_out,d_in,r,ldu,ldv,M", [
    (77, 1000, 96, 3, 3, 1),
    (77, 1000, 96, 5, 7, 3),
    (1, 1, 32, 1, 1, 1),
    (33, 17, 288, 9, 12, 8),
    (300, 2049, 320, 10, 10, 2),
    (5, 4097, 32, 4, 4, 6),
])
@pytest.mark.parametrize("align", [1, 4])  # rows kept at ldu (plain copies) or padded to 16 bytes (bulk copies)
def test_ragged_and_padded(d_out, d_in, r, ldu, ldv, M, align):
    need_gpu()
    p = synth.make_projection("ragged", d_out, d_in, r, seed=202, key=d_out * 7 + d_in, ldu=ldu, ldv=ldv)
    xb = synth.acts_bf16(synth.rng_for(203, d_in), (M, d_in))
    y = gpu_forward(p, xb, ld_align_words=align)
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
    check_tolerance(y, y_ref, S, "ragged %r" % ((d_out, d_in, r, ldu, ldv, M),))


def _unit_scales(p):
    p.s1 = np.full(p.d_out, 0x3C00, dtype=np.uint16)
    p.s2 = np.full(p.d_in, 0x3C00, dtype=np.uint16)
    return p


@pytest.mark.parametrize("d_out,d_in,r,M", [(256, 512, 128, 1), (4096, 4096, 2048, 8), (1024, 8192, 512, 2)])
def test_integer_exact_bitwise(d_out, d_in, r, M):
    need_gpu()
    p = _unit_scales(synth.make_projection("int", d_out, d_in, r, seed=204, key=d_out))
    xi = synth.rng_for(205, d_out).integers(-1, 2, size=(M, d_in)).astype(np.float32)
    xb = synth.f32_to_bf16_bits(xi)
    y = gpu_forward(p, xb)
    rows = np.arange(d_out) if d_out <= 1024 else np.linspace(0, d_out - 1, 257).astype(np.int64)
    y_ref, _ = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb, rows=rows)
    np.testing.assert_array_equal(y[:, rows], oracle.round_bf16(y_ref))


def test_per_row_magnitudes_and_zero_row():
    """Each batch row gets its own fixed-point shifts (for z and for t): rows scaled by 2^-40,
    2^-8, 1 and 2^20 (exact power-of-two scalings in bf16) and an all-zero row, in one call,
    each within its own tolerance; the zero row comes out exactly zero."""
    need_gpu()
    p = synth.make_workload("tiny")[0]
    xf = synth.rng_for(211, 5).standard_normal((5, p.d_in)).astype(np.float32)
    xf *= np.array([2.0 ** -40, 2.0 ** -8, 1.0, 2.0 ** 20, 0.0], dtype=np.float32)[:, None]
    xb = synth.f32_to_bf16_bits(xf)
    y = gpu_forward(p, xb)
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
    check_tolerance(y, y_ref, S, "per-row magnitudes")
    assert np.all(bf16_bits_to_f64(y[4]) == 0.0)


def test_every_sign_pattern_4x2_bitwise():
    """All 256 U patterns x all 256 V patterns of 4 x 2 signs, stacked into one layer
    (d_out = d_in = 1024), packed at r = 32 with pad columns that cancel exactly."""
    need_gpu()
    pats = np.array(list(itertools.product([-1, 1], repeat=8)), dtype=np.int8).reshape(256 * 4, 2)

    def words(S, pad):
        w = np.zeros(S.shape[0], dtype=np.uint32)
        for k in range(2):
            w |= (S[:, k] > 0).astype(np.uint32) << np.uint32(k)
        return (w | np.uint32(pad)).reshape(-1, 1)

    p = synth.Projection("patterns", 1024, 1024, 32, words(pats, 0xFFFFFFFC), words(pats, 0x0001FFFC),
                         np.full(1024, 0x3C00, dtype=np.uint16), np.full(1024, 0x3C00, dtype=np.uint16))
    xi = synth.rng_for(206).integers(-1, 2, size=(8, 1024)).astype(np.float32)
    xb = synth.f32_to_bf16_bits(xi)
    y = gpu_forward(p, xb)
    G = pats.astype(np.int64) @ pats.astype(np.int64).T  # rank-2 Gram of every pattern pair
    y_int = xi.astype(np.int64) @ G.T
    y_ref, _ = oracle.dense_packed(p.U, p.V, p.s1, p.s2, 32, xb)
    np.testing.assert_array_equal(y_ref, y_int.astype(np.float64))
    np.testing.assert_array_equal(y, oracle.round_bf16(y_ref))


def test_rank_one_closed_form_on_gpu():
    """Every column of U equal to u and of V equal to v: y = 32 s1 (.) u (v . (s2 (.) x))."""
    need_gpu()
    rng = np.random.default_rng(207)
    d_out, d_in = 300, 700
    u = rng.choice([-1, 1], size=d_out)
    v = rng.choice([-1, 1], size=d_in)
    p = synth.Projection("rank1", d_out, d_in, 32, np.where(u > 0, 0xFFFFFFFF, 0).astype(np.uint32)[:, None],
                         np.where(v > 0, 0xFFFFFFFF, 0).astype(np.uint32)[:, None], synth.scales_f16(rng, d_out),
                         synth.scales_f16(rng, d_in))
    xb = synth.acts_bf16(rng, (2, d_in))
    y = gpu_forward(p, xb)
    s1, s2, x = oracle.f16_to_double(p.s1), oracle.f16_to_double(p.s2), oracle.bf16_to_double(xb)
    closed = 32 * s1[None, :] * u[None, :] * (x * (s2 * v)[None, :]).sum(axis=1, keepdims=True)
    _, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, 32, xb)
    check_tolerance(y, closed, S, "rank one")


SAMPLE = 96


@pytest.mark.parametrize("workload,M", [("attn7b", 1), ("attn7b", 8), ("mlp7b", 1), ("layer70b", 1),
                                        ("layer70b", 4)])
def test_full_size_sampled_rows(workload, M):
    """Full Llama-2 shapes, launched exactly as the benchmark launches them; the oracle
    evaluates a spread of output rows (first, last and evenly spaced)."""
    need_gpu()
    for p in synth.make_workload(workload):
        xb = synth.make_input(workload, p.d_in, M, key=p.d_out)
        y = gpu_forward(p, xb)
        rows = np.unique(np.concatenate([[0, p.d_out - 1], np.linspace(0, p.d_out - 1, SAMPLE).astype(np.int64)]))
        y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb, rows=rows)
        check_tolerance(y[:, rows], y_ref, S, "%s/%s M=%d" % (workload, p.name, M))


def test_full_output_7b_every_row():
    """Every output row of the 7B attention projection (M = 2) against the oracle."""
    need_gpu()
    p = synth.make_workload("attn7b")[0]
    xb = synth.make_input("attn7b", p.d_in, 2)
    y = gpu_forward(p, xb)
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
    check_tolerance(y, y_ref, S, "attn7b all rows")


def test_run_to_run_identical():
    need_gpu()
    p = synth.make_workload("attn7b")[0]
    xb = synth.make_input("attn7b", p.d_in, 3)
    L = upload_projection(p)
    x = upload_bf16(xb)
    ys = [download_bf16_bits(nq().lrb_matvec(L, x)) for _ in range(3)]
    nq().sync_status()
    assert all(np.array_equal(ys[0], v) for v in ys[1:])


def test_workspace_reuse_across_layers_and_batches():
    """One workspace shared by calls with different layers and batch sizes on one stream."""
    need_gpu()
    ps = [synth.make_projection("a", 512, 1024, 256, seed=208, key=1),
          synth.make_projection("b", 1024, 512, 128, seed=208, key=2)]
    Ls = [upload_projection(p) for p in ps]
    need = max(L.workspace_bytes(8) for L in Ls)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    outs = []
    for rep in range(2):
        for p, L in zip(ps, Ls):
            for M in (1, 8, 3):
                xb = synth.acts_bf16(synth.rng_for(209, M, p.d_in), (M, p.d_in))
                y = nq().lrb_matvec(L, upload_bf16(xb), ws=ws)
                outs.append((p, xb, y))
    nq().sync_status()
    for p, xb, y in outs:
        y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
        check_tolerance(download_bf16_bits(y), y_ref, S, "reuse")


def test_layer_forward_dispatch_small_batch():
    need_gpu()
    p = synth.make_workload("tiny")[0]
    xb = synth.make_input("tiny", p.d_in, 4, key=9)
    y1 = gpu_forward(p, xb, fn="layer_forward")
    y2 = gpu_forward(p, xb, fn="lrb_matvec")
    np.testing.assert_array_equal(y1, y2)


def test_binding_rejects_mismatched_tensors():
    """Wrong widths, dtypes, devices or layouts raise in the binding before the library is
    called (the C ABI cannot see a tensor's extent)."""
    need_gpu()
    p = synth.make_workload("tiny")[0]
    L = upload_projection(p)
    x = upload_bf16(synth.make_input("tiny", p.d_in, 2))
    for bad in (x[:, :-8].contiguous(), x.float(), x.cpu(), x.t().contiguous().t()):
        with pytest.raises(ValueError):
            nq().layer_forward(L, bad)
    with pytest.raises(ValueError):
        nq().layer_forward(L, x, y=torch.empty((2, p.d_out - 1), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        nq().layer_forward(L, x, ws=torch.zeros(1 << 20, dtype=torch.int32, device="cuda"))
    y = nq().layer_forward(L, x)  # the same call with valid arguments runs
    nq().sync_status()
    assert tuple(y.shape) == (2, p.d_out)
