"""nq_layer_forward_group: projections sharing their input, one decode launch per stage.

Each member's output is held to the same tolerance against the oracle as a single-layer call
(2e-3 * S + 1e-5 + half a bf16 ulp).  A group of one is the single-layer path and must match
it bit for bit.  Members differ in d_out and r: the 70B q/k/v (r = 2240, 512, 512), the MLP
gate/up, and ragged tiny layers; M runs over the decode batch sizes and one prefill size.
"""
import numpy as np
import pytest
import torch

import oracle
from rank_binary_factorized_b200 import synth
from tests.gpu_util import check_tolerance, download_bf16_bits, need_gpu, nq, upload_bf16, upload_projection

pytestmark = pytest.mark.gpu


def _check_group(projs, M, seed, sample_rows=None):
    d_in = projs[0].d_in
    xb = synth.acts_bf16(synth.rng_for(seed, d_in, M), (M, d_in))
    layers = [upload_projection(p) for p in projs]
    ys = nq().layer_forward_group(layers, upload_bf16(xb))
    nq().sync_status()
    for p, y in zip(projs, ys):
        got = download_bf16_bits(y)
        rows = None if sample_rows is None else np.linspace(0, p.d_out - 1, sample_rows).astype(np.int64)
        ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb, rows=rows)
        check_tolerance(got if rows is None else got[:, rows], ref, S, "group member %s M=%d" % (p.name, M))


@pytest.mark.parametrize("M", [1, 8])
def test_group_70b_qkv(M):
    need_gpu()
    projs = synth.make_workload("layer70b")[:3]
    _check_group(projs, M, 1300 + M, sample_rows=64)


@pytest.mark.parametrize("M", [1, 2, 5, 8, 20])
def test_group_ragged_members(M):
    need_gpu()
    projs = [synth.make_projection("a", 256, 520, 128, seed=1310, key=1),
             synth.make_projection("b", 100, 520, 64, seed=1310, key=2, ldu=3, ldv=5),
             synth.make_projection("c", 300, 520, 32, seed=1310, key=3),
             synth.make_projection("d", 17, 520, 2048, seed=1310, key=4)]
    _check_group(projs, M, 1320 + M)


def test_group_70b_gate_up():
    """The 70B MLP's gate and up as the benchmark launches them: one grid of 28 word chunks in
    clusters of 4, 512-thread blocks."""
    need_gpu()
    projs = synth.make_workload("layer70b")[4:6]
    assert [p.name for p in projs] == ["gate", "up"]
    _check_group(projs, 1, 1350, sample_rows=48)


@pytest.mark.parametrize("M", [1, 8])
def test_70b_o_projection(M):
    need_gpu()
    p = synth.make_workload("layer70b")[3]
    assert p.name == "o"
    _check_group([p], M, 1360 + M, sample_rows=48)


def test_group_mlp_gate_up():
    need_gpu()
    projs = synth.make_workload("mlp7b")[:2]
    _check_group(projs, 1, 1330, sample_rows=64)


def test_group_of_one_is_the_single_layer_call():
    need_gpu()
    p = synth.make_workload("attn7b")[0]
    L = upload_projection(p)
    for M in (1, 8):
        x = upload_bf16(synth.make_input("attn7b", p.d_in, M, key=1340 + M))
        a = nq().layer_forward(L, x)
        (b,) = nq().layer_forward_group([L], x)
        nq().sync_status()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
