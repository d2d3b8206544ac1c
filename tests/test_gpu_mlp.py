"""SiLU-gated MLP block from three LRB projections (Llama-2 7B and 70B MLP shapes) and
the nq_silu_mul kernel, against the CPU oracle."""
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


@pytest.mark.parametrize("workload", ["mlp7b", "layer70b"])
def test_mlp_block_decode(workload):
    """gate, up (shared x) -> h = silu(g) * u -> down, batch 1; down outputs vs the oracle's
    MLP on a spread of rows, with S taken from the oracle's own h."""
    need_gpu()
    projs = {p.name: p for p in synth.make_workload(workload)}
    gate, up, down = projs["gate"], projs["up"], projs["down"]
    xb = synth.make_input(workload, gate.d_in, 1, key=31)
    Lg, Lu, Ld = (upload_projection(p) for p in (gate, up, down))
    x = upload_bf16(xb)
    g = nq().layer_forward(Lg, x)
    u = nq().layer_forward(Lu, x)
    h = nq().silu_mul(g, u)
    y = nq().layer_forward(Ld, h)
    nq().sync_status()
    # oracle: gate/up in the factored fp64 order, rounded to bf16, h, then the exact down
    rows = np.unique(np.concatenate([[0, down.d_out - 1], np.linspace(0, down.d_out - 1, 96).astype(np.int64)]))
    as_tuple = lambda p: (p.U, p.V, p.s1, p.s2, p.r)  # noqa: E731
    y_ref, S, _ = oracle.mlp(as_tuple(gate), as_tuple(up), as_tuple(down), xb, rows=rows, order="factored")
    check_tolerance(download_bf16_bits(y)[:, rows], y_ref, S, workload + " MLP")
