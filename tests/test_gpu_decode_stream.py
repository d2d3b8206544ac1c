"""The single-launch decode path (M <= 2, rows of U and V padded to 16 bytes) against the CPU
oracle, and the workspace state it keeps.

Page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models" (research.samsung.com
blog), section 2, factorisation equation; section 4, "Inference Performance" (binary GEMV).

- Outlier channels inside one activation row (a few channels 2^12 and 2^16 times the rest, the
  pattern of large activations in Llama hidden states) on the 7B attention and 70B q and down
  shapes, on this path and on the two-kernel path (M = 3).
- Shapes whose stage-1 stretches cross column chunks inside one CTA, partial chunks and row
  blocks, and rows of very different magnitudes in one call.
- The reserved workspace region: after any sequence of calls the barrier counter has moved by
  the grid size per single-launch call (which also shows this path ran), and the accumulator
  half and bounds the next call will use are zero.
"""
import numpy as np
import pytest
import torch

import oracle
from rank_binary_factorized_b200 import synth
from tests.gpu_util import (bf16_bits_to_f64, check_tolerance, download_bf16_bits, need_gpu, nq, upload_bf16,
                            upload_projection)

pytestmark = pytest.mark.gpu

RESERVED = 4096 + 512 * 1024  # NQ_WS_RESERVED_BYTES


def _sm_count():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _reserved_state(ws):
    """Barrier counter, the bounds of both halves and the accumulator halves of the reserved
    region: counters at bytes 0..7, bounds [2][4][2] int64 from byte 64, halves of 256 KiB each
    from byte 4096."""
    head = ws[:RESERVED].cpu().numpy()
    counter = int(head[:8].view(np.uint64)[0])
    bounds = head[64:64 + 2 * 4 * 2 * 8].view(np.int64).reshape(2, 8)
    halves = head[4096:].view(np.int64).reshape(2, -1)
    return counter, bounds, halves


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


@pytest.mark.parametrize("d_out,d_in,r,M", [
    (777, 3000, 1056, 2),   # 33 words: three chunks, the last one word wide
    (1000, 20000, 544, 1),  # many row blocks per chunk, stretches cross chunks
    (33, 65, 32, 2),        # one chunk, one partial row block
    (4099, 257, 2016, 1),   # 63 words, d_out not a multiple of a block
])
def test_ragged_single_launch(d_out, d_in, r, M):
    need_gpu()
    p = synth.make_projection("ragged1", d_out, d_in, r, seed=2200, key=d_out + d_in)
    xb = synth.acts_bf16(synth.rng_for(2201, d_in, M), (M, d_in))
    L = upload_projection(p)
    y = download_bf16_bits(nq().lrb_matvec(L, upload_bf16(xb)))
    nq().sync_status()
    y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
    check_tolerance(y, y_ref, S, "single launch %r" % ((d_out, d_in, r, M),))


def test_rows_of_very_different_magnitude_and_zero_input():
    """Each batch row has its own common exponent: rows scaled by 2^-40 and 2^20 in one call; a
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


def test_reserved_region_is_ready_after_calls():
    """After single, grouped and two-kernel calls on one workspace, the barrier counter has
    advanced by the grid size once per single-launch call, and the accumulator half and bounds
    that the next call will use are zero."""
    need_gpu()
    G = _sm_count()
    projs = synth.make_workload("layer70b")
    layers = [upload_projection(p) for p in projs]
    need = max(nq().group_workspace_bytes(layers[:3], 2), max(L.workspace_bytes(3) for L in layers))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    x = upload_bf16(synth.make_input("layer70b", 8192, 2, key=2400))
    calls = 0
    for rep in range(2):
        nq().layer_forward_group(layers[:3], x, ws=ws)      # q, k, v: one launch
        calls += 1
        nq().layer_forward(layers[3], x, ws=ws)             # o
        calls += 1
        nq().layer_forward(layers[3], x[:1], ws=ws)         # o at M = 1
        calls += 1
        x3 = upload_bf16(synth.make_input("layer70b", 8192, 3, key=2401))
        nq().layer_forward(layers[3], x3, ws=ws)            # M = 3: the two-kernel path
        nq().sync_status()
        counter, bounds, halves = _reserved_state(ws)
        assert counter == calls * G
        nxt = calls & 1
        assert not halves[nxt].any() and not bounds[nxt].any()
