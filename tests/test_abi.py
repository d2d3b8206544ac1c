"""The C ABI: libnq.so loads, exports every entry point include/nq.h declares, and rejects
bad arguments on the host with the documented status before anything is launched.

No compute call runs here: every call below fails validation (or, on a machine without a
GPU, the device check), so no pointer is ever dereferenced.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nq.h")

NQ = dict(OK=0, NULL=1, SHAPE=2, ALIGN=3, WORKSPACE=4, DEVICE=5, LAUNCH=6, TIMEOUT=7, SCRATCH_LIMIT=8)
NOALLOC_SCRATCH_BYTES = 2 * 1024 * 1024  # NQ_NOALLOC_SCRATCH_BYTES in include/nq.h


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"NQ_API\s+[\w\s\*]+?\b(nq_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def nq():
    from rank_binary_factorized_b200 import nq as mod
    return mod


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for name in ["nq_pack_signs", "nq_lrb_matvec", "nq_lrb_matmul", "nq_layer_forward", "nq_workspace_bytes",
                 "nq_silu_mul", "nq_sync_status", "nq_status_string"]:
        assert name in syms


def test_library_exports_every_declared_symbol(nq):
    lib = ctypes.CDLL(nq.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    # and nothing else with the nq_ prefix leaks out undocumented
    out = os.popen("nm -D --defined-only %s" % nq.LIB_PATH).read()
    exported = set(re.findall(r" T (nq_\w+)", out))
    assert exported == set(declared_symbols())


def test_status_strings_and_version(nq):
    for code, name in nq.STATUS_NAMES.items():
        assert nq.status_string(code).startswith(name)
    assert "sm_100a" in nq.version()


def _layer(nq, d_out=64, d_in=96, r=64, ldu=None, ldv=None, U=0x10000, V=0x20000, s1=0x30000, s2=0x40000):
    return nq.nq_lrb_layer(d_out, d_in, r, U, ldu if ldu is not None else r // 32, V,
                           ldv if ldv is not None else r // 32, s1, s2)


def _call(nq, fn, L, x=0x50000, y=0x60000, M=1, ws=0x70000, ws_bytes=1 << 30):
    lib = nq.raw_lib()
    return getattr(lib, fn)(ctypes.byref(L) if L is not None else None, x, y, M, ws, ws_bytes, None)


@pytest.mark.parametrize("fn", ["nq_lrb_matvec", "nq_lrb_matmul", "nq_layer_forward", "nq_lrb_transposed"])
def test_forward_argument_errors(nq, fn):
    assert _call(nq, fn, None) == NQ["NULL"]
    assert _call(nq, fn, _layer(nq, U=0)) == NQ["NULL"]
    assert _call(nq, fn, _layer(nq), x=0) == NQ["NULL"]
    assert _call(nq, fn, _layer(nq), ws=0) == NQ["NULL"]
    assert _call(nq, fn, _layer(nq, r=48)) == NQ["SHAPE"]  # r % 32 != 0
    assert _call(nq, fn, _layer(nq, r=0)) == NQ["SHAPE"]
    assert _call(nq, fn, _layer(nq, d_out=0)) == NQ["SHAPE"]
    assert _call(nq, fn, _layer(nq, d_in=-3)) == NQ["SHAPE"]
    assert _call(nq, fn, _layer(nq, ldu=1)) == NQ["SHAPE"]  # ld below r/32
    assert _call(nq, fn, _layer(nq, ldv=1)) == NQ["SHAPE"]
    assert _call(nq, fn, _layer(nq, r=262144 + 32, ldu=8193, ldv=8193)) == NQ["SHAPE"]  # above NQ_MAX_RANK_LIMIT
    assert _call(nq, fn, _layer(nq), M=0) == NQ["SHAPE"]
    assert _call(nq, fn, _layer(nq, V=0x20004)) == NQ["ALIGN"]
    assert _call(nq, fn, _layer(nq), x=0x50002) == NQ["ALIGN"]
    assert _call(nq, fn, _layer(nq), ws_bytes=16) == NQ["WORKSPACE"]


def test_scale_grads_argument_errors(nq):
    lib = nq.raw_lib()

    def call(L, x=0x50000, ybar=0x60000, M=1, g1=0x80000, g2=0x90000, ws=0x70000, ws_bytes=1 << 30):
        return lib.nq_lrb_scale_grads(ctypes.byref(L) if L is not None else None, x, ybar, M, g1, g2, ws, ws_bytes,
                                      None)

    assert call(None) == NQ["NULL"]
    assert call(_layer(nq, V=0)) == NQ["NULL"]
    assert call(_layer(nq), ybar=0) == NQ["NULL"]
    assert call(_layer(nq), g1=0) == NQ["NULL"]
    assert call(_layer(nq), g2=0) == NQ["NULL"]
    assert call(_layer(nq, r=48)) == NQ["SHAPE"]
    assert call(_layer(nq), M=0) == NQ["SHAPE"]
    assert call(_layer(nq), g2=0x90004) == NQ["ALIGN"]
    assert call(_layer(nq), x=0x50008) == NQ["ALIGN"]
    assert call(_layer(nq), ws_bytes=16) == NQ["WORKSPACE"]


def test_sign_grads_argument_errors(nq):
    lib = nq.raw_lib()

    def call(L, x=0x50000, ybar=0x60000, M=1, gU=0x80000, ldgu=64, gV=0x90000, ldgv=64, ws=0x70000, ws_bytes=1 << 30):
        return lib.nq_lrb_sign_grads(ctypes.byref(L) if L is not None else None, x, ybar, M, gU, ldgu, gV, ldgv, ws,
                                     ws_bytes, None)

    assert call(None) == NQ["NULL"]
    assert call(_layer(nq, U=0)) == NQ["NULL"]
    assert call(_layer(nq), x=0) == NQ["NULL"]
    assert call(_layer(nq), gU=0) == NQ["NULL"]
    assert call(_layer(nq), gV=0) == NQ["NULL"]
    assert call(_layer(nq, r=48)) == NQ["SHAPE"]
    assert call(_layer(nq), M=0) == NQ["SHAPE"]
    assert call(_layer(nq), ldgu=32) == NQ["SHAPE"]  # below r
    assert call(_layer(nq), ldgv=60) == NQ["SHAPE"]
    assert call(_layer(nq), ldgu=66) == NQ["ALIGN"]  # row stride not a multiple of 16 bytes
    assert call(_layer(nq), gV=0x90008) == NQ["ALIGN"]
    assert call(_layer(nq), ws_bytes=16) == NQ["WORKSPACE"]
    for M in (1, 8, 9, 2048):
        assert lib.nq_sign_grads_workspace_bytes(ctypes.byref(_layer(nq, d_out=28672, d_in=8192, r=3520)), M) > 0
    assert lib.nq_sign_grads_workspace_bytes(ctypes.byref(_layer(nq)), 0) == 0
    assert lib.nq_sign_grads_workspace_bytes(ctypes.byref(_layer(nq, r=48)), 1) == 0


def test_selftest_argument_errors(nq):
    lib = nq.raw_lib()
    assert lib.nq_selftest_bounded_wait(999, None) == NQ["SHAPE"]
    assert lib.nq_selftest_bounded_wait(2000001, None) == NQ["SHAPE"]


def test_workspace_covers_both_directions(nq):
    """One workspace serves the forward product, the transpose and the scale gradients: the
    size is the same for a layer and for the layer with its two sides exchanged."""
    lib = nq.raw_lib()
    for M in (1, 8, 64, 2048):
        a = lib.nq_workspace_bytes(ctypes.byref(_layer(nq, d_out=28672, d_in=8192, r=3520)), M)
        b = lib.nq_workspace_bytes(ctypes.byref(_layer(nq, d_out=8192, d_in=28672, r=3520)), M)
        assert a == b > 0


def test_from_latent_argument_errors(nq):
    lib = nq.raw_lib()

    def call(Uh=0x10000, ld_uh=64, Vh=0x20000, ld_vh=64, d_out=8, d_in=8, r=64, U=0x30000, ldu=2, V=0x40000, ldv=2,
             s1=0x50000, s2=0x60000, eta=0, ws=0x70000, ws_bytes=1 << 20):
        return lib.nq_lrb_from_latent(Uh, ld_uh, Vh, ld_vh, d_out, d_in, r, U, ldu, V, ldv, s1, s2, eta, ws, ws_bytes,
                                      None)

    assert call(r=48) == NQ["SHAPE"]
    assert call(ld_uh=32) == NQ["SHAPE"]
    assert call(ldv=1) == NQ["SHAPE"]
    assert call(d_in=0) == NQ["SHAPE"]
    assert call(Uh=0) == NQ["NULL"]
    assert call(s2=0) == NQ["NULL"]
    assert call(V=0x40004) == NQ["ALIGN"]
    assert call(eta=0x80004) == NQ["ALIGN"]
    assert call(ws_bytes=16) == NQ["WORKSPACE"]
    assert lib.nq_from_latent_workspace_bytes(8, 8, 64, 2, 2) > 0
    assert lib.nq_from_latent_workspace_bytes(8, 8, 48, 2, 2) == 0


def test_group_argument_errors(nq):
    lib = nq.raw_lib()
    Ls = [_layer(nq), _layer(nq, d_out=32, r=32), _layer(nq, d_in=64)]
    arr = (ctypes.POINTER(nq.nq_lrb_layer) * 3)(*[ctypes.pointer(L) for L in Ls])
    ys = (ctypes.c_void_p * 3)(0x60000, 0x61000, 0x62000)
    assert lib.nq_layer_forward_group(arr, 2, 0x50000, ys, 1, 0x70000, 1 << 30, None) != NQ["SHAPE"]
    assert lib.nq_layer_forward_group(arr, 3, 0x50000, ys, 1, 0x70000, 1 << 30, None) == NQ["SHAPE"]  # d_in differs
    assert lib.nq_layer_forward_group(arr, 0, 0x50000, ys, 1, 0x70000, 1 << 30, None) == NQ["SHAPE"]
    assert lib.nq_layer_forward_group(arr, 5, 0x50000, ys, 1, 0x70000, 1 << 30, None) == NQ["SHAPE"]
    assert lib.nq_layer_forward_group(arr, 2, 0x50000, ys, 1, 0x70000, 16, None) == NQ["WORKSPACE"]
    assert lib.nq_group_workspace_bytes(arr, 2, 1) > 0
    assert lib.nq_group_workspace_bytes(arr, 3, 1) == 0


def test_matvec_rejects_large_batch(nq):
    assert _call(nq, "nq_lrb_matvec", _layer(nq), M=nq.MATVEC_MAX_M + 1) == NQ["SHAPE"]


def test_workspace_bytes(nq):
    lib = nq.raw_lib()
    L = _layer(nq)
    for M in (1, 8, 9, 64, 2048):
        assert lib.nq_workspace_bytes(ctypes.byref(L), M) > 0
    assert lib.nq_workspace_bytes(ctypes.byref(L), 0) == 0
    assert lib.nq_workspace_bytes(ctypes.byref(_layer(nq, r=40)), 1) == 0


def test_pack_argument_errors(nq):
    lib = nq.raw_lib()
    assert lib.nq_pack_signs(0x1000, 4, 48, 48, 0x2000, 2, None) == NQ["SHAPE"]  # r % 32
    assert lib.nq_pack_signs(0x1000, 4, 64, 32, 0x2000, 2, None) == NQ["SHAPE"]  # ld_latent < r
    assert lib.nq_pack_signs(0x1000, 4, 64, 64, 0x2000, 1, None) == NQ["SHAPE"]  # ld_words < r/32
    assert lib.nq_pack_signs(0x1000, -1, 64, 64, 0x2000, 2, None) == NQ["SHAPE"]
    assert lib.nq_pack_signs(0x1000, 0, 64, 64, 0x2000, 2, None) == NQ["OK"]  # empty: no-op
    assert lib.nq_pack_signs(0, 4, 64, 64, 0x2000, 2, None) == NQ["NULL"]
    assert lib.nq_pack_signs(0x1000, 4, 64, 64, 0, 2, None) == NQ["NULL"]
    assert lib.nq_pack_signs(0x1004, 4, 64, 64, 0x2000, 2, None) == NQ["ALIGN"]


def test_silu_argument_errors(nq):
    lib = nq.raw_lib()
    assert lib.nq_silu_mul(0x1000, 0x2000, 0x3000, -1, None) == NQ["SHAPE"]
    assert lib.nq_silu_mul(0x1000, 0x2000, 0x3000, 0, None) == NQ["OK"]
    assert lib.nq_silu_mul(0, 0x2000, 0x3000, 8, None) == NQ["NULL"]
    assert lib.nq_silu_mul(0x1000, 0x2002, 0x3000, 8, None) == NQ["ALIGN"]


def test_no_gpu_gives_device_error(nq):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; this checks the CPU-only path")
    # valid arguments, no device: the call must refuse, not fall back to anything
    assert _call(nq, "nq_lrb_matvec", _layer(nq)) == NQ["DEVICE"]
    assert nq.raw_lib().nq_pack_signs(0x1000, 4, 64, 64, 0x2000, 2, None) == NQ["DEVICE"]


def _noalloc(nq):
    fn = nq.raw_lib().nq_lrb_matvec_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(nq.nq_lrb_layer), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                   ctypes.c_void_p]
    return lambda L, x=0x50000, y=0x60000, M=1: fn(ctypes.byref(L) if L is not None else None, x, y, M, None)


def test_noalloc_validates_like_matvec(nq):
    """The allocation-free entry point refuses what nq_lrb_matvec refuses, with the same status."""
    na = _noalloc(nq)
    cases = [
        (None, {}), (_layer(nq, r=48), {}), (_layer(nq, ldu=1), {}), (_layer(nq, U=0), {}),
        (_layer(nq, s2=0x40002), {}), (_layer(nq, d_out=0), {}),
        (_layer(nq), dict(M=0)), (_layer(nq), dict(M=9)), (_layer(nq), dict(x=0)), (_layer(nq), dict(y=0)),
        (_layer(nq), dict(x=0x50008)), (_layer(nq), dict(y=0x60002)),
        (_layer(nq, r=1 << 17), dict(M=8)),
    ]
    for L, kw in cases:
        want = _call(nq, "nq_lrb_matvec", L, **kw)
        assert want != NQ["OK"]
        assert na(L, **kw) == want, (L and (L.d_out, L.d_in, L.r), kw)


def test_noalloc_scratch_covers_every_accepted_decode_shape(nq):
    """For every M the decode path takes, the largest rank r it accepts (stage 2's shared
    memory caps it) still fits the static scratch: the call gets past the scratch check to the
    device check, and one step of r further both entry points refuse the shape."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; accepted shapes would launch")
    na = _noalloc(nq)
    lib = nq.raw_lib()
    for M in range(1, 9):
        lo, hi = 32, 1 << 22  # lo accepted, hi refused
        assert na(_layer(nq, r=lo), M=M) == NQ["DEVICE"]
        assert na(_layer(nq, r=hi), M=M) == NQ["SHAPE"]
        while hi - lo > 32:
            mid = (lo + hi) // 64 * 32
            if na(_layer(nq, r=mid), M=M) == NQ["SHAPE"]:
                hi = mid
            else:
                lo = mid
        L = _layer(nq, r=lo)
        assert na(L, M=M) == NQ["DEVICE"], M  # not NQ_ERR_SCRATCH_LIMIT
        assert _call(nq, "nq_lrb_matvec", L, M=M) == NQ["DEVICE"]
        assert _call(nq, "nq_lrb_matvec", _layer(nq, r=hi), M=M) == NQ["SHAPE"]
        need = lib.nq_workspace_bytes(ctypes.byref(_layer(nq, d_out=64, d_in=64, r=lo)), M)
        assert 0 < need <= NOALLOC_SCRATCH_BYTES, (M, lo, need)


def test_mlp_gate_up_argument_errors(nq):
    lib = nq.raw_lib()
    fn = lib.nq_mlp_gate_up
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(nq.nq_lrb_layer), ctypes.POINTER(nq.nq_lrb_layer), ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    wsb = lib.nq_mlp_gate_up_workspace_bytes
    wsb.restype = ctypes.c_size_t
    wsb.argtypes = [ctypes.POINTER(nq.nq_lrb_layer), ctypes.POINTER(nq.nq_lrb_layer), ctypes.c_int64]
    g, u = _layer(nq, d_out=64, d_in=96, r=64), _layer(nq, d_out=64, d_in=96, r=96)

    def call(gl=g, ul=u, x=0x50000, h=0x60000, M=1, ws=0x70000, ws_bytes=1 << 30):
        return fn(ctypes.byref(gl) if gl is not None else None, ctypes.byref(ul) if ul is not None else None,
                  x, h, M, ws, ws_bytes, None)

    assert call(gl=None) == NQ["NULL"]
    assert call(ul=_layer(nq, d_out=64, d_in=97, r=64)) == NQ["SHAPE"]   # d_in differs
    assert call(ul=_layer(nq, d_out=65, d_in=96, r=64)) == NQ["SHAPE"]   # d_out differs
    assert call(M=0) == NQ["SHAPE"]
    assert call(ul=_layer(nq, d_out=64, d_in=96, r=1 << 17)) == NQ["SHAPE"]  # too large for decode
    assert call(x=0) == NQ["NULL"] and call(h=0) == NQ["NULL"] and call(ws=0) == NQ["NULL"]
    assert call(x=0x50008) == NQ["ALIGN"]
    assert call(ws_bytes=16) == NQ["WORKSPACE"]
    assert wsb(ctypes.byref(g), ctypes.byref(_layer(nq, d_out=65, d_in=96, r=64)), 1) == 0
    assert wsb(ctypes.byref(g), ctypes.byref(u), 0) == 0
    for M in (1, 8, 9, 512):
        need = wsb(ctypes.byref(g), ctypes.byref(u), M)
        assert need >= 2 * M * 64 * 2  # room for the unfused gate and up outputs
    import torch
    if not torch.cuda.is_available():
        assert call() == NQ["DEVICE"]


def test_binding_refuses_host_tensors_before_any_call(nq):
    """The binding checks tensor arguments before their addresses reach the library (which
    reads device memory only): host tensors and wrong types raise, nothing is launched."""
    import torch
    U, V = torch.zeros((64, 2), dtype=torch.int32), torch.zeros((96, 2), dtype=torch.int32)
    s1, s2 = torch.zeros(64, dtype=torch.float16), torch.zeros(96, dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA"):
        nq.Layer(U, V, s1, s2, 64)
    with pytest.raises(TypeError):
        nq.Layer(None, V, s1, s2, 64)
    with pytest.raises(ValueError, match="CUDA"):
        nq.pack_signs(torch.zeros((4, 64)))
    with pytest.raises(ValueError, match="CUDA"):
        nq.silu_mul(torch.zeros(8, dtype=torch.bfloat16), torch.zeros(8, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):
        nq.lrb_from_latent(torch.zeros((8, 64)), torch.zeros((8, 64)))
