"""Edge cases of the decode path (nq_lrb_matvec) against the CPU oracle.

Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models" (research.samsung.com
blog), section 2, factorisation equation; section 4, "Inference Performance" (binary GEMV).

- Outlier channels inside one activation row (a few channels 2^12 and 2^16 times the rest, the
  pattern of large activations in Llama hidden states) on the 7B attention and 70B q and down
  shapes: x is quantised to fixed point per row slice of V, so the small channels of a slice
  with an outlier keep fewer bits; the tolerance still holds because S contains the outlier's
  own terms.
- Ragged shapes (partial word chunks, partial row slices, d_out not a multiple of a tile) and
  rows of very different magnitudes in one call, with an all-zero input giving exactly zero.
"""
import numpy as np
import pytest

import oracle
from rank_binary_factorized_b200 import synth
from tests.gpu_util import (bf16_bits_to_f64, check_tolerance, download_bf16_bits, half_ulp_bf16, need_gpu, nq,
                            upload_bf16, upload_projection)

pytestmark = pytest.mark.gpu

def _outlier_input(d_in, M, seed, factors):
    rng = synth.rng_for(seed, d_in, M)
    xf = rng.standard_normal((M, d_in)).astype(np.float32)
    cols = rng.choice(d_in, size=len(factors), replace=False)
    for m in range(M):
        xf[m, cols] *= np.array(factors, dtype=np.float32)  # powers of two: exact in bf16
    return synth.f32_to_bf16_bits(xf)


@pytest.mark.parametrize("workload,name", [("attn7b", "q"), ("layer70b", "q"), ("layer70b", "down")])
@pytest.mark.parametrize("M", [1, 2, 3])
def test_outlier_channels_in_one_row(workload, name, M):
    need_gpu()
    projs = {p.name: p for p in synth.make_workload(workload)}
    p = projs.get(name) or synth.make_workload(workload)[0]
    xb = _outlier_input(p.d_in, M, 2100 + M, [2.0 ** 12, 2.0 ** 16, 2.0 ** 16, 2.0 ** 12])
    L = upload_projection(p)
    y = download_bf16_bits(nq().lrb_matvec(L, upload_bf16(xb)))
    nq().sync_status()
    rows = np.unique(np.concatenate([[0, p.d_out - 1], np.linspace(0, p.d_out - 1, 128).astype(np.int64)]))
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb, rows=rows)
    check_tolerance(y[:, rows], y_ref, S, "outliers %s/%s M=%d" % (workload, p.name, M))
    # Where the outliers dominate (|y| >= S/2) the stated bound 2e-3 S is below one bf16 unit of
    # y, so only the output rounding can use it up: the arithmetic before it (fixed-point z and
    # t) must leave y within one bf16 unit of the exact value.
    got = bf16_bits_to_f64(y[:, rows])
    dom = np.abs(y_ref) >= 0.5 * S
    assert dom.sum() >= 8
    assert np.all(np.abs(got - y_ref)[dom] <= 2.0 * half_ulp_bf16(y_ref[dom]))


@pytest.mark.parametrize("d_out,d_in,r,M", [
    (777, 3000, 1056, 2),   # 33 words: three chunks, the last one word wide
    (1000, 20000, 544, 1),  # long row slices
    (33, 65, 32, 2),        # one word chunk, one partial row slice
    (4099, 257, 2016, 1),   # 63 words, d_out not a multiple of a tile
])
def test_ragged_shapes(d_out, d_in, r, M):
    need_gpu()
    p = synth.make_projection("ragged1", d_out, d_in, r, seed=2200, key=d_out + d_in)
    xb = synth.acts_bf16(synth.rng_for(2201, d_in, M), (M, d_in))
    L = upload_projection(p)
    y = download_bf16_bits(nq().lrb_matvec(L, upload_bf16(xb)))
    nq().sync_status()
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
    check_tolerance(y, y_ref, S, "ragged %r" % ((d_out, d_in, r, M),))


def test_rows_of_very_different_magnitude_and_zero_input():
    """Each batch row has its own fixed-point shifts: rows scaled by 2^-40 and 2^20 in one call; a
    second call with an all-zero x gives exactly zero."""
    need_gpu()
    p = synth.make_workload("attn7b")[0]
    xf = synth.rng_for(2300).standard_normal((2, p.d_in)).astype(np.float32)
    xf *= np.array([2.0 ** -40, 2.0 ** 20], dtype=np.float32)[:, None]
    xb = synth.f32_to_bf16_bits(xf)
    L = upload_projection(p)
    y = download_bf16_bits(nq().lrb_matvec(L, upload_bf16(xb)))
    z = download_bf16_bits(nq().lrb_matvec(L, upload_bf16(np.zeros((1, p.d_in), dtype=np.uint16))))
    nq().sync_status()
    rows = np.linspace(0, p.d_out - 1, 200).astype(np.int64)
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb, rows=rows)
    check_tolerance(y[:, rows], y_ref, S, "row magnitudes 2^-40, 2^20")
    assert np.all(bf16_bits_to_f64(z) == 0.0)


@pytest.mark.parametrize("d_out,d_in,r,M,align", [
    (200, 64, 20224, 1, 4),     # largest rank at M = 1: a single chunk buffer
    (3000, 96, 16384, 1, 4),    # two one-tile buffers, each block's chunks alternating in them
    (60000, 64, 256, 1, 4),     # 26 M-tiles per block: the ring of six buffers wraps around
    (60000, 64, 224, 2, 1),     # the same with rows of 7 words, copied in 4-byte pieces
    (60001, 48, 320, 3, 1),     # 10 words (8-byte pieces), d_out odd: the last s1 half alone
    (100, 64, 7168, 8, 4),      # largest rank at M = 8 (three B-table column tiles)
])
def test_stage2_ring_regimes(d_out, d_in, r, M, align):
    """Stage 2 streams U through a ring of chunk buffers whose depth and chunk size depend on
    r, M and d_out: these shapes cover a single buffer, buffers reused many times, and the
    4- and 8-byte copy paths of unpadded strides, on sampled rows (first and last included)."""
    need_gpu()
    p = synth.make_projection("ring", d_out, d_in, r, seed=2300, key=d_out + r)
    xb = synth.acts_bf16(synth.rng_for(2301, d_in, M), (M, d_in))
    L = upload_projection(p, ld_align_words=align)
    y = download_bf16_bits(nq().lrb_matvec(L, upload_bf16(xb)))
    nq().sync_status()
    rows = np.unique(np.concatenate([[0, 1, d_out - 2, d_out - 1], np.linspace(0, d_out - 1, 200).astype(np.int64)]))
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb, rows=rows)
    check_tolerance(y[:, rows], y_ref, S, "ring regime %r" % ((d_out, d_in, r, M, align),))
