"""SiLU-gated MLP block from three LRB projections (Llama-2 7B and 70B MLP shapes): the
nq_silu_mul kernel and the fused gate/up call nq_mlp_gate_up, against the CPU oracle and, bit for
bit, against the unfused calls they replace."""
import numpy as np
import pytest

import oracle
from rank_binary_factorized_b200 import synth
from tests.gpu_util import check_tolerance, download_bf16_bits, need_gpu, nq, upload_bf16, upload_projection

pytestmark = pytest.mark.gpu


def test_silu_mul_within_one_bf16_ulp():
    """fp32 math on the GPU vs fp64 in the oracle: the two roundings to bf16 may land one
    unit in the last place apart, never more."""
    need_gpu()
    rng = synth.rng_for(301)
    n = 100_003  # not a multiple of the 8-element vector width
    gb = synth.f32_to_bf16_bits((4 * rng.standard_normal(n)).astype(np.float32))
    ub = synth.acts_bf16(rng, n)
    h = nq().silu_mul(upload_bf16(gb), upload_bf16(ub))
    nq().sync_status()
    got = download_bf16_bits(h).astype(np.int32)
    want = oracle.silu_mul(oracle.bf16_to_double(gb), oracle.bf16_to_double(ub)).astype(np.int32)
    # compare as ordered integers (same sign): at most one unit apart
    gs = np.where(got & 0x8000, -(got & 0x7FFF), got)
    ws_ = np.where(want & 0x8000, -(want & 0x7FFF), want)
    assert np.abs(gs - ws_).max() <= 1


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("workload", ["mlp7b", "layer70b"])
def test_mlp_block_decode(workload, fused):
    """gate, up (shared x) -> h = silu(g) * u -> down, batch 1; down outputs vs the oracle's
    MLP on a spread of rows, with S taken from the oracle's own h.  fused: h from
    nq_mlp_gate_up instead of two projections and nq_silu_mul."""
    need_gpu()
    projs = {p.name: p for p in synth.make_workload(workload)}
    gate, up, down = projs["gate"], projs["up"], projs["down"]
    xb = synth.make_input(workload, gate.d_in, 1, key=31)
    Lg, Lu, Ld = (upload_projection(p) for p in (gate, up, down))
    x = upload_bf16(xb)
    if fused:
        h = nq().mlp_gate_up(Lg, Lu, x)
    else:
        g = nq().layer_forward(Lg, x)
        u = nq().layer_forward(Lu, x)
        h = nq().silu_mul(g, u)
    y = nq().layer_forward(Ld, h)
    nq().sync_status()
    # oracle: gate/up in the factored fp64 order, rounded to bf16, h, then the exact down
    rows = np.unique(np.concatenate([[0, down.d_out - 1], np.linspace(0, down.d_out - 1, 96).astype(np.int64)]))
    as_tuple = lambda p: (p.U, p.V, p.s1, p.s2, p.r)  # noqa: E731
    y_ref, S, _ = oracle.mlp(as_tuple(gate), as_tuple(up), as_tuple(down), xb, rows=rows, order="factored")
    check_tolerance(download_bf16_bits(y)[:, rows], y_ref, S, workload + " MLP" + (" fused" if fused else ""))


def _gate_up_pair(d_out, d_in, r_gate, r_up, seed):
    gate = synth.make_projection("gate", d_out, d_in, r_gate, seed=seed, key=1)
    up = synth.make_projection("up", d_out, d_in, r_up, seed=seed, key=2)
    return gate, up


@pytest.mark.parametrize("d_out,d_in,r_gate,r_up,M", [
    (11008, 4096, 2368, 2368, 1),   # 7B MLP
    (11008, 4096, 2368, 2368, 3),
    (11008, 4096, 2368, 2368, 8),
    (28672, 8192, 3520, 3520, 1),   # 70B MLP
    (28672, 8192, 3520, 3520, 2),
    (1000, 300, 96, 160, 1),        # ragged: d_out not a multiple of 16, different ranks
    (1000, 300, 96, 160, 5),
    (37, 64, 32, 64, 2),            # a single partial M-tile
    (300, 64, 12000, 12000, 1),     # both stage-2 tables too large together: the unfused decode path
    (2000, 512, 256, 320, 9),       # prefill path
    (2000, 512, 256, 320, 64),
])
def test_mlp_gate_up_equals_unfused_calls(d_out, d_in, r_gate, r_up, M):
    """nq_mlp_gate_up == nq_layer_forward_group({gate, up}) then nq_silu_mul, bit for bit, on
    every element (the same integer sums and the same bf16 roundings of g and u)."""
    need_gpu()
    gate, up = _gate_up_pair(d_out, d_in, r_gate, r_up, seed=330 + M)
    xb = synth.acts_bf16(synth.rng_for(331, d_in, M), (M, d_in))
    Lg, Lu = upload_projection(gate), upload_projection(up)
    x = upload_bf16(xb)
    g, u = nq().layer_forward_group([Lg, Lu], x)
    h_ref = nq().silu_mul(g, u)
    h = nq().mlp_gate_up(Lg, Lu, x)
    h2 = nq().mlp_gate_up(Lg, Lu, x)  # again, on the workspace the first call left behind
    nq().sync_status()
    want = download_bf16_bits(h_ref)
    assert np.array_equal(download_bf16_bits(h), want)
    assert np.array_equal(download_bf16_bits(h2), want)
