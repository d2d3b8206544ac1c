"""nq_lrb_matvec_noalloc: the decode entry point for callers that cannot allocate device
memory (engine plug-ins handed only their tensors, allocator-free C callers).  Its scratch is
a static array inside libnq.so.

Called here through the C ABI with ctypes, twice in a row per layer (the second call runs on
the scratch the first one left behind).  It runs the same kernels as nq_lrb_matvec -- the
entry point that takes a caller workspace -- so its output must equal that one's bit for bit
on every row, and, like every decode result, lie within the parity tolerance of the CPU
oracle on sampled rows.  This file is collected last so that a run stopping at the first
failure has already run every other test; it also passes on its own in a fresh process (the
first call does the per-device set-up).
"""
import ctypes

import numpy as np
import pytest

import oracle
from rank_binary_factorized_b200 import synth
from tests.gpu_util import (REL, ABS, bf16_bits_to_f64, download_bf16_bits, half_ulp_bf16, need_gpu, nq,
                            upload_bf16, upload_projection)

pytestmark = pytest.mark.gpu

NQ_ERR_SHAPE = 2


def noalloc_fn():
    mod = nq()
    fn = mod.raw_lib().nq_lrb_matvec_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(mod.nq_lrb_layer), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                   ctypes.c_void_p]
    return fn


@pytest.mark.parametrize("workload,M", [("tiny", 1), ("attn7b", 1), ("attn7b", 8), ("layer70b", 1)])
def test_noalloc_matches_workspace_entry_point_on_two_calls(workload, M):
    need_gpu()
    import torch
    mod = nq()
    fn = noalloc_fn()
    projs = synth.make_workload(workload)
    p = projs[-1]  # layer70b: the down projection (d_in = 28672, the largest stage 1)
    L = upload_projection(p)
    stream = torch.cuda.current_stream()
    for call in range(2):
        xb = synth.make_input(workload, p.d_in, M, key=500 + call)
        x = upload_bf16(xb)
        y_ws = mod.lrb_matvec(L, x)  # existing entry point, caller workspace
        y_na = torch.empty_like(y_ws)
        st = fn(ctypes.byref(L.struct), x.data_ptr(), y_na.data_ptr(), M, ctypes.c_void_p(stream.cuda_stream))
        assert st == 0, mod.status_string(st)
        mod.sync_status()
        got_bits = download_bf16_bits(y_na)
        want_bits = download_bf16_bits(y_ws)
        # the same kernels on the same input: identical bits on every row
        assert np.array_equal(got_bits, want_bits), "call %d differs from nq_lrb_matvec" % call
        # and the oracle's bound on a spread of rows (first and last included)
        rows = np.unique(np.concatenate([[0, p.d_out - 1], np.linspace(0, p.d_out - 1, 64).astype(np.int64)]))
        y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb, rows=rows)
        got = bf16_bits_to_f64(got_bits)[:, rows]
        assert np.all(np.abs(got - y_ref) <= REL * S + ABS + half_ulp_bf16(y_ref)), "call %d vs the oracle" % call


def test_noalloc_refuses_oversize_layers_like_matvec():
    """A layer too large for the decode kernels (r = 131072 at M = 8: stage 2's digit table
    of t alone would be 3 MiB) is refused by both entry points with the same status, before
    anything is launched: y keeps its contents."""
    need_gpu()
    mod = nq()
    fn = noalloc_fn()
    M = 8
    p = synth.make_projection("big", 64, 64, 131072, seed=501)
    L = upload_projection(p)
    x = upload_bf16(synth.acts_bf16(synth.rng_for(502), (M, p.d_in)))
    fill = np.full((M, p.d_out), 0x3F80, dtype=np.uint16)  # bf16 1.0
    y = upload_bf16(fill)
    st = fn(ctypes.byref(L.struct), x.data_ptr(), y.data_ptr(), M, None)
    assert st == NQ_ERR_SHAPE, mod.status_string(st)
    with pytest.raises(mod.NQError) as err:
        mod.lrb_matvec(L, x)
    assert err.value.status == NQ_ERR_SHAPE
    mod.sync_status()
    assert np.array_equal(download_bf16_bits(y), fill)
