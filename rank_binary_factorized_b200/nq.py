"""Thin Python binding of libnq.so (include/nq.h) -- argument marshalling only.

Every step of the LRB path runs in the CUDA library; this module checks tensor arguments
(CUDA device, dtype, shape, layout: the C ABI cannot see a tensor's extent), turns them into
device pointers and the current torch stream into a ``cudaStream_t``.  PyTorch provides
device memory and streams, nothing else.  If ``libnq.so`` is missing the import fails: there
is no other implementation to fall back to.

Tensor conventions (device tensors, contiguous):
  packed signs  int32 [rows][ld] (the bits of uint32 words)
  s1, s2        float16 [d_out], [d_in]
  x, y          bfloat16 [M][d_in], [M][d_out]
  latent        float32 [rows][ld_latent]
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libnq.so is not built (python -m rank_binary_factorized_b200.build): " + LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)

NQ_OK = 0
STATUS_NAMES = {0: "NQ_OK", 1: "NQ_ERR_NULL", 2: "NQ_ERR_SHAPE", 3: "NQ_ERR_ALIGN", 4: "NQ_ERR_WORKSPACE",
                5: "NQ_ERR_DEVICE", 6: "NQ_ERR_LAUNCH", 7: "NQ_ERR_TIMEOUT"}
MATVEC_MAX_M = 8

_i64 = ctypes.c_int64
_p = ctypes.c_void_p


class nq_lrb_layer(ctypes.Structure):
    _fields_ = [("d_out", _i64), ("d_in", _i64), ("r", _i64), ("U", _p), ("ldu", _i64), ("V", _p), ("ldv", _i64),
                ("s1", _p), ("s2", _p)]


_lib.nq_pack_signs.restype = ctypes.c_int
_lib.nq_pack_signs.argtypes = [_p, _i64, _i64, _i64, _p, _i64, _p]
_lib.nq_workspace_bytes.restype = ctypes.c_size_t
_lib.nq_workspace_bytes.argtypes = [ctypes.POINTER(nq_lrb_layer), _i64]
for _name in ("nq_lrb_matvec", "nq_lrb_matmul", "nq_layer_forward"):
    getattr(_lib, _name).restype = ctypes.c_int
    getattr(_lib, _name).argtypes = [ctypes.POINTER(nq_lrb_layer), _p, _p, _i64, _p, ctypes.c_size_t, _p]
_lib.nq_silu_mul.restype = ctypes.c_int
_lib.nq_silu_mul.argtypes = [_p, _p, _p, _i64, _p]
_lib.nq_lrb_transposed.restype = ctypes.c_int
_lib.nq_lrb_transposed.argtypes = [ctypes.POINTER(nq_lrb_layer), _p, _p, _i64, _p, ctypes.c_size_t, _p]
_lib.nq_from_latent_workspace_bytes.restype = ctypes.c_size_t
_lib.nq_from_latent_workspace_bytes.argtypes = [_i64, _i64, _i64, _i64, _i64]
_lib.nq_lrb_from_latent.restype = ctypes.c_int
_lib.nq_lrb_from_latent.argtypes = [_p, _i64, _p, _i64, _i64, _i64, _i64, _p, _i64, _p, _i64, _p, _p, _p, _p,
                                    ctypes.c_size_t, _p]
_lib.nq_mlp_gate_up_workspace_bytes.restype = ctypes.c_size_t
_lib.nq_mlp_gate_up_workspace_bytes.argtypes = [ctypes.POINTER(nq_lrb_layer), ctypes.POINTER(nq_lrb_layer), _i64]
_lib.nq_mlp_gate_up.restype = ctypes.c_int
_lib.nq_mlp_gate_up.argtypes = [ctypes.POINTER(nq_lrb_layer), ctypes.POINTER(nq_lrb_layer), _p, _p, _i64, _p,
                                ctypes.c_size_t, _p]
_lib.nq_group_workspace_bytes.restype = ctypes.c_size_t
_lib.nq_group_workspace_bytes.argtypes = [ctypes.POINTER(ctypes.POINTER(nq_lrb_layer)), ctypes.c_int, _i64]
_lib.nq_layer_forward_group.restype = ctypes.c_int
_lib.nq_layer_forward_group.argtypes = [ctypes.POINTER(ctypes.POINTER(nq_lrb_layer)), ctypes.c_int, _p,
                                        ctypes.POINTER(_p), _i64, _p, ctypes.c_size_t, _p]
_lib.nq_lrb_scale_grads.restype = ctypes.c_int
_lib.nq_lrb_scale_grads.argtypes = [ctypes.POINTER(nq_lrb_layer), _p, _p, _i64, _p, _p, _p, ctypes.c_size_t, _p]
_lib.nq_sync_status.restype = ctypes.c_int
_lib.nq_sign_grads_workspace_bytes.restype = ctypes.c_size_t
_lib.nq_sign_grads_workspace_bytes.argtypes = [ctypes.POINTER(nq_lrb_layer), _i64]
_lib.nq_lrb_sign_grads.restype = ctypes.c_int
_lib.nq_lrb_sign_grads.argtypes = [ctypes.POINTER(nq_lrb_layer), _p, _p, _i64, _p, _i64, _p, _i64, _p, ctypes.c_size_t,
                                   _p]
_lib.nq_selftest_bounded_wait.restype = ctypes.c_int
_lib.nq_selftest_bounded_wait.argtypes = [_i64, _p]
_lib.nq_sync_status.argtypes = [_p]
_lib.nq_status_string.restype = ctypes.c_char_p
_lib.nq_status_string.argtypes = [ctypes.c_int]
_lib.nq_version.restype = ctypes.c_char_p
_lib.nq_version.argtypes = []


class NQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__("%s: %s" % (fn, _lib.nq_status_string(status).decode()))


def _check(fn: str, status: int) -> None:
    if status != NQ_OK:
        raise NQError(fn, status)


def version() -> str:
    return _lib.nq_version().decode()


def status_string(status: int) -> str:
    return _lib.nq_status_string(status).decode()


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _need(t, name: str, dtype, shape=None, device=None, contiguous: bool = True) -> None:
    """Checks a tensor argument before its address reaches the library, which reads device
    memory only and at the layout nq.h states: a CUDA tensor of the given dtype (and shape and
    device), contiguous unless the call takes a row stride."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s: expected a torch.Tensor, got %s" % (name, type(t).__name__))
    if not t.is_cuda:
        raise ValueError("%s: expected a CUDA tensor, got one on %s" % (name, t.device))
    if t.dtype != dtype:
        raise ValueError("%s: expected dtype %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(int(d) for d in shape):
        raise ValueError("%s: expected shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if device is not None and t.device != device:
        raise ValueError("%s: on %s, the layer's tensors on %s" % (name, t.device, device))
    if contiguous and not t.is_contiguous():
        raise ValueError("%s: expected a contiguous tensor" % name)


def _need_rows(t, name: str, dtype, rows: int, min_cols: int, device=None) -> None:
    """A 2-D CUDA tensor with `rows` rows of at least `min_cols` columns and unit column stride
    (the call takes its row stride)."""
    _need(t, name, dtype, device=device, contiguous=False)
    if t.dim() != 2 or int(t.shape[0]) != rows or int(t.shape[1]) < min_cols or t.stride(1) != 1:
        raise ValueError("%s: expected [%d][>= %d] with unit column stride, got shape %s strides %s" %
                         (name, rows, min_cols, tuple(t.shape), tuple(t.stride())))


def _need_ws(ws, layer_device) -> None:
    _need(ws, "ws", torch.uint8, device=layer_device)


class Layer:
    """A device-resident LRB layer: packed U, V (int32 words), fp16 s1, s2."""

    def __init__(self, U: torch.Tensor, V: torch.Tensor, s1: torch.Tensor, s2: torch.Tensor, r: int):
        _need(U, "U", torch.int32)
        if U.dim() != 2:
            raise ValueError("U: expected [d_out][ldu] words, got shape %s" % (tuple(U.shape),))
        _need(V, "V", torch.int32, device=U.device)
        if V.dim() != 2:
            raise ValueError("V: expected [d_in][ldv] words, got shape %s" % (tuple(V.shape),))
        _need(s1, "s1", torch.float16, shape=(U.shape[0],), device=U.device)
        _need(s2, "s2", torch.float16, shape=(V.shape[0],), device=U.device)
        self.U, self.V, self.s1, self.s2 = U, V, s1, s2
        self.d_out, self.ldu = int(U.shape[0]), int(U.shape[1])
        self.d_in, self.ldv = int(V.shape[0]), int(V.shape[1])
        self.r = int(r)
        self.struct = nq_lrb_layer(self.d_out, self.d_in, self.r, _ptr(U), self.ldu, _ptr(V), self.ldv, _ptr(s1),
                                   _ptr(s2))
        self._ws = {}

    @classmethod
    def from_host(cls, U, V, s1_bits, s2_bits, r: int, device="cuda", ld_align_words: int = 4) -> "Layer":
        """From numpy arrays: uint32 words and fp16 bit patterns (uint16).  Rows of U and V are
        padded with zero words to a multiple of `ld_align_words` words: at the default 4 (16
        bytes) the tensor-core path loads the packed signs by TMA; any stride works."""
        import numpy as np

        def dev(a, dt):
            return torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(device)

        def words(a):
            a = np.ascontiguousarray(a)
            nw = a.shape[1]
            ld = -(-nw // ld_align_words) * ld_align_words
            if ld != nw:
                b = np.zeros((a.shape[0], ld), dtype=a.dtype)
                b[:, :nw] = a
                a = b
            return dev(a, np.int32)

        return cls(words(U), words(V), dev(s1_bits, np.float16), dev(s2_bits, np.float16), r)

    def workspace_bytes(self, M: int) -> int:
        return int(_lib.nq_workspace_bytes(ctypes.byref(self.struct), M))

    def workspace(self, M: int) -> torch.Tensor:
        """A zero-filled workspace large enough for M rows, cached on the layer and grown on
        demand.  Every call on this layer that passes no ``ws`` uses it, so calls that may run
        at the same time on the GPU (on different streams) must each pass their own ``ws``."""
        need = self.workspace_bytes(M)
        if need == 0:
            raise NQError("nq_workspace_bytes", 2)
        ws = self._ws.get("ws")
        if ws is None or ws.numel() < need:
            ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=self.U.device)
            self._ws["ws"] = ws
        return ws

    @property
    def storage_bytes(self) -> int:
        return 4 * (self.d_out + self.d_in) * self.r // 32 + 2 * (self.d_out + self.d_in)


def pack_signs(latent: torch.Tensor, r: int | None = None, ld_words: int | None = None, out=None,
               stream=None) -> torch.Tensor:
    """sign(latent) >= 0 packed 32 per word along r (bit k%32 of word k/32)."""
    _need(latent, "latent", torch.float32, contiguous=False)
    if latent.dim() != 2 or latent.stride(1) != 1:
        raise ValueError("latent must be a 2-D float32 tensor with unit column stride")
    rows, ld_latent = int(latent.shape[0]), int(latent.stride(0))
    r = int(latent.shape[1]) if r is None else int(r)
    if r > int(latent.shape[1]):
        raise ValueError("r = %d exceeds the latent's %d columns" % (r, int(latent.shape[1])))
    ld_words = r // 32 if ld_words is None else int(ld_words)
    if out is None:
        out = torch.empty((rows, ld_words), dtype=torch.int32, device=latent.device)
    _need(out, "out", torch.int32, shape=(rows, ld_words), device=latent.device)
    _check("nq_pack_signs", _lib.nq_pack_signs(_ptr(latent), rows, r, ld_latent, _ptr(out), ld_words,
                                               _stream_ptr(stream)))
    return out


def _forward(fn_name: str, layer: Layer, x: torch.Tensor, y=None, ws=None, stream=None) -> torch.Tensor:
    dev = layer.U.device
    _need(x, "x", torch.bfloat16, device=dev)
    M = int(x.shape[0])
    _need(x, "x", torch.bfloat16, shape=(M, layer.d_in))
    if y is None:
        y = torch.empty((M, layer.d_out), dtype=torch.bfloat16, device=x.device)
    _need(y, "y", torch.bfloat16, shape=(M, layer.d_out), device=dev)
    if ws is None:
        ws = layer.workspace(M)
    _need_ws(ws, dev)
    fn = getattr(_lib, fn_name)
    _check(fn_name, fn(ctypes.byref(layer.struct), _ptr(x), _ptr(y), M, _ptr(ws), ws.numel(), _stream_ptr(stream)))
    return y


def lrb_matvec(layer: Layer, x: torch.Tensor, y=None, ws=None, stream=None) -> torch.Tensor:
    return _forward("nq_lrb_matvec", layer, x, y, ws, stream)


def lrb_matmul(layer: Layer, x: torch.Tensor, y=None, ws=None, stream=None) -> torch.Tensor:
    return _forward("nq_lrb_matmul", layer, x, y, ws, stream)


def layer_forward(layer: Layer, x: torch.Tensor, y=None, ws=None, stream=None) -> torch.Tensor:
    return _forward("nq_layer_forward", layer, x, y, ws, stream)


def lrb_transposed(layer: Layer, ybar: torch.Tensor, xbar=None, ws=None, stream=None) -> torch.Tensor:
    """xbar = the layer's transpose applied to ybar ([M][d_out] bf16 -> [M][d_in] bf16)."""
    dev = layer.U.device
    _need(ybar, "ybar", torch.bfloat16, device=dev)
    M = int(ybar.shape[0])
    _need(ybar, "ybar", torch.bfloat16, shape=(M, layer.d_out))
    if xbar is None:
        xbar = torch.empty((M, layer.d_in), dtype=torch.bfloat16, device=ybar.device)
    _need(xbar, "xbar", torch.bfloat16, shape=(M, layer.d_in), device=dev)
    if ws is None:
        ws = layer.workspace(M)
    _need_ws(ws, dev)
    _check("nq_lrb_transposed", _lib.nq_lrb_transposed(ctypes.byref(layer.struct), _ptr(ybar), _ptr(xbar), M,
                                                       _ptr(ws), ws.numel(), _stream_ptr(stream)))
    return xbar


def lrb_scale_grads(layer: Layer, x: torch.Tensor, ybar: torch.Tensor, ws=None, stream=None):
    """(dL/ds1 [d_out], dL/ds2 [d_in]) fp32 for L = sum <ybar, layer(x)>."""
    dev = layer.U.device
    _need(x, "x", torch.bfloat16, device=dev)
    M = int(x.shape[0])
    _need(x, "x", torch.bfloat16, shape=(M, layer.d_in))
    _need(ybar, "ybar", torch.bfloat16, shape=(M, layer.d_out), device=dev)
    g1 = torch.empty(layer.d_out, dtype=torch.float32, device=x.device)
    g2 = torch.empty(layer.d_in, dtype=torch.float32, device=x.device)
    if ws is None:
        ws = layer.workspace(M)
    _need_ws(ws, dev)
    _check("nq_lrb_scale_grads", _lib.nq_lrb_scale_grads(ctypes.byref(layer.struct), _ptr(x), _ptr(ybar), M,
                                                         _ptr(g1), _ptr(g2), _ptr(ws), ws.numel(),
                                                         _stream_ptr(stream)))
    return g1, g2


def sign_grads_workspace_bytes(layer: Layer, M: int) -> int:
    n = int(_lib.nq_sign_grads_workspace_bytes(ctypes.byref(layer.struct), int(M)))
    if n == 0:
        raise NQError("nq_sign_grads_workspace_bytes", 2)
    return n


def lrb_sign_grads(layer: Layer, x: torch.Tensor, ybar: torch.Tensor, gU=None, gV=None, ws=None, stream=None):
    """(dL/dU [d_out][r], dL/dV [d_in][r]) fp32 for L = sum <ybar, layer(x)>: the gradients the
    identity straight-through estimator passes to the latent factors.  gU, gV may be given
    ([rows][ld] fp32 with ld >= r a multiple of 4); only their first r columns are written."""
    dev = layer.U.device
    _need(x, "x", torch.bfloat16, device=dev)
    M = int(x.shape[0])
    _need(x, "x", torch.bfloat16, shape=(M, layer.d_in))
    _need(ybar, "ybar", torch.bfloat16, shape=(M, layer.d_out), device=dev)
    r = layer.r
    if gU is None:
        gU = torch.empty((layer.d_out, r), dtype=torch.float32, device=x.device)
    if gV is None:
        gV = torch.empty((layer.d_in, r), dtype=torch.float32, device=x.device)
    _need_rows(gU, "gU", torch.float32, layer.d_out, r, device=dev)
    _need_rows(gV, "gV", torch.float32, layer.d_in, r, device=dev)
    if ws is None:
        ws = torch.empty(sign_grads_workspace_bytes(layer, M), dtype=torch.uint8, device=x.device)
    _need_ws(ws, dev)
    _check("nq_lrb_sign_grads", _lib.nq_lrb_sign_grads(ctypes.byref(layer.struct), _ptr(x), _ptr(ybar), M, _ptr(gU),
                                                       gU.stride(0), _ptr(gV), gV.stride(0), _ptr(ws), ws.numel(),
                                                       _stream_ptr(stream)))
    return gU, gV


def lrb_from_latent(Uh: torch.Tensor, Vh: torch.Tensor, r: int | None = None, ld_align_words: int = 4,
                    stream=None):
    """A device Layer from fp32 latent proxies Uh [d_out][r], Vh [d_in][r]: magnitude balancing,
    mean-absolute-value scales, packed signs.  Returns (Layer, eta as a 0-d fp64 tensor)."""
    r = int(Uh.shape[1]) if r is None else int(r)
    _need_rows(Uh, "Uh", torch.float32, int(Uh.shape[0]), r)
    _need_rows(Vh, "Vh", torch.float32, int(Vh.shape[0]), r, device=Uh.device)
    d_out, d_in = int(Uh.shape[0]), int(Vh.shape[0])
    ld = -(-(r // 32) // ld_align_words) * ld_align_words
    dev = Uh.device
    U = torch.empty((d_out, ld), dtype=torch.int32, device=dev)
    V = torch.empty((d_in, ld), dtype=torch.int32, device=dev)
    s1 = torch.empty(d_out, dtype=torch.float16, device=dev)
    s2 = torch.empty(d_in, dtype=torch.float16, device=dev)
    eta = torch.empty((), dtype=torch.float64, device=dev)
    need = int(_lib.nq_from_latent_workspace_bytes(d_out, d_in, r, ld, ld))
    if need == 0:
        raise NQError("nq_from_latent_workspace_bytes", 2)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    _check("nq_lrb_from_latent", _lib.nq_lrb_from_latent(_ptr(Uh), int(Uh.stride(0)), _ptr(Vh), int(Vh.stride(0)),
                                                         d_out, d_in, r, _ptr(U), ld, _ptr(V), ld, _ptr(s1),
                                                         _ptr(s2), _ptr(eta), _ptr(ws), need, _stream_ptr(stream)))
    return Layer(U, V, s1, s2, r), eta


def _layer_array(layers):
    arr = (ctypes.POINTER(nq_lrb_layer) * len(layers))()
    for i, L in enumerate(layers):
        arr[i] = ctypes.pointer(L.struct)
    return arr


def group_workspace_bytes(layers, M: int) -> int:
    return int(_lib.nq_group_workspace_bytes(_layer_array(layers), len(layers), M))


def layer_forward_group(layers, x: torch.Tensor, ys=None, ws=None, stream=None):
    """y_l = layers[l](x) for projections sharing x (one decode launch per stage for M <= 8)."""
    if len(layers) == 0:
        raise ValueError("layers: expected at least one layer")
    dev = layers[0].U.device
    _need(x, "x", torch.bfloat16, device=dev)
    M = int(x.shape[0])
    for L in layers:
        if L.U.device != dev:
            raise ValueError("layers: all on one device")
        _need(x, "x", torch.bfloat16, shape=(M, L.d_in))
    if ys is None:
        ys = [torch.empty((M, L.d_out), dtype=torch.bfloat16, device=x.device) for L in layers]
    if len(ys) != len(layers):
        raise ValueError("ys: expected one output per layer")
    for i, (L, y) in enumerate(zip(layers, ys)):
        _need(y, "ys[%d]" % i, torch.bfloat16, shape=(M, L.d_out), device=dev)
    if ws is None:
        need = group_workspace_bytes(layers, M)
        if need == 0:
            raise NQError("nq_group_workspace_bytes", 2)
        ws = torch.zeros(need, dtype=torch.uint8, device=x.device)
    _need_ws(ws, dev)
    yp = (_p * len(ys))(*[_ptr(y) for y in ys])
    _check("nq_layer_forward_group", _lib.nq_layer_forward_group(_layer_array(layers), len(layers), _ptr(x), yp, M,
                                                                 _ptr(ws), ws.numel(), _stream_ptr(stream)))
    return ys


def mlp_gate_up_workspace_bytes(gate: Layer, up: Layer, M: int) -> int:
    return int(_lib.nq_mlp_gate_up_workspace_bytes(ctypes.byref(gate.struct), ctypes.byref(up.struct), M))


def mlp_gate_up(gate: Layer, up: Layer, x: torch.Tensor, h=None, ws=None, stream=None) -> torch.Tensor:
    """h = bf16(silu(bf16(gate x)) * bf16(up x)) ([M][d_out] bf16), SiLU.mul fused into decode."""
    dev = gate.U.device
    if up.U.device != dev:
        raise ValueError("gate, up: expected one device")
    _need(x, "x", torch.bfloat16, device=dev)
    M = int(x.shape[0]) if x.dim() == 2 else -1
    _need(x, "x", torch.bfloat16, shape=(M, gate.d_in), device=dev)
    if h is None:
        h = torch.empty((M, gate.d_out), dtype=torch.bfloat16, device=dev)
    _need(h, "h", torch.bfloat16, shape=(M, gate.d_out), device=dev)
    if ws is None:
        need = mlp_gate_up_workspace_bytes(gate, up, M)
        if need == 0:
            raise NQError("nq_mlp_gate_up_workspace_bytes", 2)
        ws = torch.zeros(need, dtype=torch.uint8, device=dev)
    _need_ws(ws, dev)
    _check("nq_mlp_gate_up", _lib.nq_mlp_gate_up(ctypes.byref(gate.struct), ctypes.byref(up.struct), _ptr(x), _ptr(h),
                                                 M, _ptr(ws), ws.numel(), _stream_ptr(stream)))
    return h


def silu_mul(g: torch.Tensor, u: torch.Tensor, h=None, stream=None) -> torch.Tensor:
    _need(g, "g", torch.bfloat16)
    _need(u, "u", torch.bfloat16, shape=tuple(g.shape), device=g.device)
    if h is None:
        h = torch.empty_like(g)
    _need(h, "h", torch.bfloat16, shape=tuple(g.shape), device=g.device)
    _check("nq_silu_mul", _lib.nq_silu_mul(_ptr(g), _ptr(u), _ptr(h), g.numel(), _stream_ptr(stream)))
    return h


def selftest_bounded_wait(limit_us: int = 20000, stream=None) -> None:
    """Launch the diagnostic kernel whose bounded wait runs out (see nq.h); the next
    sync_status raises NQError with NQ_ERR_TIMEOUT."""
    _check("nq_selftest_bounded_wait", _lib.nq_selftest_bounded_wait(int(limit_us), _stream_ptr(stream)))


def sync_status(stream=None) -> None:
    _check("nq_sync_status", _lib.nq_sync_status(_stream_ptr(stream)))


def raw_lib() -> ctypes.CDLL:
    """The loaded libnq.so (for callers that marshal arguments themselves)."""
    return _lib
