"""CPU oracle for the low-rank binary (LRB) matmul -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package.  The product path (``rank_binary_factorized_b200``) never imports it
and shares no code with it; the C source ``nq_oracle.c`` is compiled into its own
``liboracle.so`` with gcc.

Every function cites the passage it follows on the page "NanoQuant: Efficient Sub-1-Bit
Quantization of Large Language Models" (research.samsung.com blog):

* section 2, "Low-Rank Binary Factorization", the factorisation equation
  ``W ~= s1 (.) (U V^T) (.) s2^T`` and the storage sentence after it;
* section 3, "Step 3: Factorized Component Refinement", the use of sign(U), sign(V);
* section 3, "Phase 3: Scale-Only Model Reconstruction", packing frozen signs into integers.

Where the page is silent (sign(0), bit order, dtypes, the MLP composition) the readings are
the ones documented in ``nq_oracle.c``'s header.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compiles ``nq_oracle.c`` into ``liboracle.so`` (plain gcc, no SIMD flags)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        # NQ_ORACLE_SO points the wrapper at another build of nq_oracle.c (used by the
        # mutation test, which checks that the pins fail on a deliberately broken copy).
        L = ctypes.CDLL(os.environ.get("NQ_ORACLE_SO") or build())
        L.nq_oracle_f16_to_double.restype = ctypes.c_double
        L.nq_oracle_f16_to_double.argtypes = [ctypes.c_uint16]
        L.nq_oracle_bf16_to_double.restype = ctypes.c_double
        L.nq_oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.nq_oracle_double_to_bf16.restype = ctypes.c_uint16
        L.nq_oracle_double_to_bf16.argtypes = [ctypes.c_double]
        L.nq_oracle_f16_array_to_double.restype = None
        L.nq_oracle_f16_array_to_double.argtypes = [_p, _i64, _p]
        L.nq_oracle_bf16_array_to_double.restype = None
        L.nq_oracle_bf16_array_to_double.argtypes = [_p, _i64, _p]
        L.nq_oracle_pack.restype = ctypes.c_int
        L.nq_oracle_pack.argtypes = [_p, _i64, _i64, _i64, _p, _i64]
        L.nq_oracle_unpack.restype = ctypes.c_int
        L.nq_oracle_unpack.argtypes = [_p, _i64, _i64, _i64, _p]
        L.nq_oracle_gram_signs.restype = None
        L.nq_oracle_gram_signs.argtypes = [_p, _p, _i64, _i64, _i64, _p]
        L.nq_oracle_gram_packed.restype = None
        L.nq_oracle_gram_packed.argtypes = [_p, _i64, _p, _i64, _i64, _i64, _i64, _p]
        L.nq_oracle_dense_signs.restype = None
        L.nq_oracle_dense_signs.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _p, _i64, _p, _p]
        L.nq_oracle_dense_packed.restype = ctypes.c_int
        L.nq_oracle_dense_packed.argtypes = [_p, _i64, _p, _i64, _p, _p, _i64, _i64, _i64, _p, _i64,
                                             _p, _i64, _p, _p]
        L.nq_oracle_factored_packed.restype = ctypes.c_int
        L.nq_oracle_factored_packed.argtypes = [_p, _i64, _p, _i64, _p, _p, _i64, _i64, _i64, _p, _i64, _p]
        L.nq_oracle_transposed_packed.restype = ctypes.c_int
        L.nq_oracle_transposed_packed.argtypes = [_p, _i64, _p, _i64, _p, _p, _i64, _i64, _i64, _p, _i64,
                                                  _p, _i64, _p, _p]
        L.nq_oracle_scale_grads_packed.restype = ctypes.c_int
        L.nq_oracle_scale_grads_packed.argtypes = [_p, _i64, _p, _i64, _p, _p, _i64, _i64, _i64, _p, _p, _i64,
                                                   _p, _p, _p, _p]
        L.nq_oracle_sign_grads_packed.restype = ctypes.c_int
        L.nq_oracle_sign_grads_packed.argtypes = [_p, _i64, _p, _i64, _p, _p, _i64, _i64, _i64, _p, _p, _i64,
                                                  _p, _i64, _p, _i64, _p, _i64, _p, _p, _p, _p]
        L.nq_oracle_double_to_f16.restype = ctypes.c_uint16
        L.nq_oracle_double_to_f16.argtypes = [ctypes.c_double]
        L.nq_oracle_from_latent.restype = ctypes.c_int
        L.nq_oracle_from_latent.argtypes = [_p, _i64, _p, _i64, _i64, _i64, _i64, _p, _i64, _p, _i64, _p, _p, _p,
                                            _p, _p]
        L.nq_oracle_silu_mul.restype = None
        L.nq_oracle_silu_mul.argtypes = [_p, _p, _i64, _p]
        L.nq_oracle_round_bf16.restype = None
        L.nq_oracle_round_bf16.argtypes = [_p, _i64, _p]
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# ----------------------------------------------------------------------------- formats
def f16_to_double(bits) -> np.ndarray:
    """IEEE binary16 bit patterns -> fp64 (exact)."""
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    lib().nq_oracle_f16_array_to_double(_ptr(b), b.size, _ptr(out))
    return out


def bf16_to_double(bits) -> np.ndarray:
    """bfloat16 bit patterns -> fp64 (exact)."""
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    lib().nq_oracle_bf16_array_to_double(_ptr(b), b.size, _ptr(out))
    return out


def round_bf16(values) -> np.ndarray:
    """fp64 -> bfloat16 bit patterns, round to nearest even, straight from fp64."""
    v = _c(values, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().nq_oracle_round_bf16(_ptr(v), v.size, _ptr(out))
    return out


# ----------------------------------------------------------------------------- signs
def pack(latent, r: int | None = None, ld_words: int | None = None) -> np.ndarray:
    """sign(latent) packed 32 per uint32 along r, LSB first, bit 1 for latent >= 0.

    Follows section 3 ("Step 3" sign(U), sign(V); "Phase 3" packing) with the readings in
    the C header: +0, -0 -> +1, NaN -> -1, pad words 0.
    """
    L = _c(latent, np.float32)
    rows, ld = L.shape
    r = ld if r is None else r
    ld_words = r // 32 if ld_words is None else ld_words
    out = np.empty((rows, ld_words), dtype=np.uint32)
    rc = lib().nq_oracle_pack(_ptr(L), rows, r, ld, _ptr(out), ld_words)
    if rc != 0:
        raise ValueError("nq_oracle_pack: bad sizes")
    return out


def unpack(packed, r: int) -> np.ndarray:
    """Packed words [rows][ld] -> int8 signs [rows][r] (+1 for bit 1)."""
    P = _c(packed, np.uint32)
    rows, ld = P.shape
    out = np.empty((rows, r), dtype=np.int8)
    rc = lib().nq_oracle_unpack(_ptr(P), rows, r, ld, _ptr(out))
    if rc != 0:
        raise ValueError("nq_oracle_unpack: bad sizes")
    return out


def gram_signs(U, V) -> np.ndarray:
    """G = U V^T by the literal triple loop on int8 signs."""
    U = _c(U, np.int8)
    V = _c(V, np.int8)
    G = np.empty((U.shape[0], V.shape[0]), dtype=np.int32)
    lib().nq_oracle_gram_signs(_ptr(U), _ptr(V), U.shape[0], V.shape[0], U.shape[1], _ptr(G))
    return G


def gram_packed(Uw, Vw, r: int) -> np.ndarray:
    """G = U V^T from packed rows: r - 2 * popcount(u XOR v)."""
    Uw = _c(Uw, np.uint32)
    Vw = _c(Vw, np.uint32)
    G = np.empty((Uw.shape[0], Vw.shape[0]), dtype=np.int32)
    lib().nq_oracle_gram_packed(_ptr(Uw), Uw.shape[1], _ptr(Vw), Vw.shape[1], Uw.shape[0], Vw.shape[0], r,
                                _ptr(G))
    return G


# ----------------------------------------------------------------------------- forward
def dense_signs(U, V, s1, s2, x):
    """The definition W_ij = s1_i (sum_k U_ik V_jk) s2_j, y = x W^T, S = sum_j |W_ij x_j|.

    Section 2, "Low-Rank Binary Factorization" (factorisation equation), on unpacked int8
    signs and fp64 values.  ``x`` is [B][d_in]; returns (y, S), each [B][d_out].
    """
    U = _c(U, np.int8)
    V = _c(V, np.int8)
    s1 = _c(s1, np.float64)
    s2 = _c(s2, np.float64)
    x = _c(np.atleast_2d(x), np.float64)
    d_out, r = U.shape
    d_in = V.shape[0]
    B = x.shape[0]
    y = np.empty((B, d_out), dtype=np.float64)
    S = np.empty((B, d_out), dtype=np.float64)
    lib().nq_oracle_dense_signs(_ptr(U), _ptr(V), _ptr(s1), _ptr(s2), d_out, d_in, r, _ptr(x), B, _ptr(y),
                                _ptr(S))
    return y, S


def dense_packed(Uw, Vw, s1_f16, s2_f16, r: int, x_bf16, rows=None):
    """The definition on the packed layout (fp16 scale bits, bf16 activation bits).

    Section 2 factorisation equation; the Gram entry is taken from packed words.  ``rows``
    selects output rows (all when None).  Returns (y, S), each [B][n_rows], fp64.
    """
    Uw = _c(Uw, np.uint32)
    Vw = _c(Vw, np.uint32)
    s1 = _c(s1_f16, np.uint16)
    s2 = _c(s2_f16, np.uint16)
    x = _c(np.atleast_2d(x_bf16), np.uint16)
    d_out, d_in, B = Uw.shape[0], Vw.shape[0], x.shape[0]
    if rows is None:
        rows_arr = None
        n = d_out
    else:
        rows_arr = _c(rows, np.int64)
        n = rows_arr.size
    y = np.empty((B, n), dtype=np.float64)
    S = np.empty((B, n), dtype=np.float64)
    rc = lib().nq_oracle_dense_packed(_ptr(Uw), Uw.shape[1], _ptr(Vw), Vw.shape[1], _ptr(s1), _ptr(s2), d_out,
                                      d_in, r, _ptr(x), B, None if rows_arr is None else _ptr(rows_arr), n,
                                      _ptr(y), _ptr(S))
    if rc != 0:
        raise ValueError("nq_oracle_dense_packed failed (%d)" % rc)
    return y, S


def transposed_packed(Uw, Vw, s1_f16, s2_f16, r: int, ybar_bf16, cols=None):
    """The layer's transpose, xbar[b][j] = sum_i W_ij ybar[b][i] (Phase 3 scale-only
    calibration backpropagates through the frozen factors), on the packed layout.  ``cols``
    selects output columns j (all d_in when None).  Returns (xbar, S), each [B][n_cols]."""
    Uw = _c(Uw, np.uint32)
    Vw = _c(Vw, np.uint32)
    s1 = _c(s1_f16, np.uint16)
    s2 = _c(s2_f16, np.uint16)
    yb = _c(np.atleast_2d(ybar_bf16), np.uint16)
    d_out, d_in, B = Uw.shape[0], Vw.shape[0], yb.shape[0]
    cols_arr = None if cols is None else _c(cols, np.int64)
    n = d_in if cols is None else cols_arr.size
    xbar = np.empty((B, n), dtype=np.float64)
    S = np.empty((B, n), dtype=np.float64)
    rc = lib().nq_oracle_transposed_packed(_ptr(Uw), Uw.shape[1], _ptr(Vw), Vw.shape[1], _ptr(s1), _ptr(s2), d_out,
                                           d_in, r, _ptr(yb), B, None if cols_arr is None else _ptr(cols_arr), n,
                                           _ptr(xbar), _ptr(S))
    if rc != 0:
        raise ValueError("nq_oracle_transposed_packed failed (%d)" % rc)
    return xbar, S


def scale_grads_packed(Uw, Vw, s1_f16, s2_f16, r: int, x_bf16, ybar_bf16):
    """dL/ds1 and dL/ds2 for L = sum_b <ybar_b, y_b>, with the magnitudes of their terms.
    Returns (g1 [d_out], S1 [d_out], g2 [d_in], S2 [d_in]), fp64."""
    Uw = _c(Uw, np.uint32)
    Vw = _c(Vw, np.uint32)
    s1 = _c(s1_f16, np.uint16)
    s2 = _c(s2_f16, np.uint16)
    x = _c(np.atleast_2d(x_bf16), np.uint16)
    yb = _c(np.atleast_2d(ybar_bf16), np.uint16)
    d_out, d_in, B = Uw.shape[0], Vw.shape[0], x.shape[0]
    if yb.shape != (B, d_out) or x.shape != (B, d_in):
        raise ValueError("x must be [B][d_in] and ybar [B][d_out]")
    g1, S1 = np.empty(d_out), np.empty(d_out)
    g2, S2 = np.empty(d_in), np.empty(d_in)
    rc = lib().nq_oracle_scale_grads_packed(_ptr(Uw), Uw.shape[1], _ptr(Vw), Vw.shape[1], _ptr(s1), _ptr(s2), d_out,
                                            d_in, r, _ptr(x), _ptr(yb), B, _ptr(g1), _ptr(S1), _ptr(g2), _ptr(S2))
    if rc != 0:
        raise ValueError("nq_oracle_scale_grads_packed failed (%d)" % rc)
    return g1, S1, g2, S2


def sign_grads_packed(Uw, Vw, s1_f16, s2_f16, r: int, x_bf16, ybar_bf16, rows_u=None, rows_v=None, ks=None):
    """dL/dU and dL/dV (the gradients the identity straight-through estimator hands to the
    latent factors) for L = sum_b <ybar_b, y_b>, with the magnitudes of their terms.
    ``rows_u``, ``rows_v`` and ``ks`` select rows of U, rows of V and rank columns (all when
    None).  Returns (gU, SU [n_rows_u][n_ks], gV, SV [n_rows_v][n_ks]), fp64."""
    Uw = _c(Uw, np.uint32)
    Vw = _c(Vw, np.uint32)
    s1 = _c(s1_f16, np.uint16)
    s2 = _c(s2_f16, np.uint16)
    x = _c(np.atleast_2d(x_bf16), np.uint16)
    yb = _c(np.atleast_2d(ybar_bf16), np.uint16)
    d_out, d_in, B = Uw.shape[0], Vw.shape[0], x.shape[0]
    if yb.shape != (B, d_out) or x.shape != (B, d_in):
        raise ValueError("x must be [B][d_in] and ybar [B][d_out]")
    ru = None if rows_u is None else _c(rows_u, np.int64)
    rv = None if rows_v is None else _c(rows_v, np.int64)
    kk = None if ks is None else _c(ks, np.int64)
    nu = d_out if ru is None else ru.size
    nv = d_in if rv is None else rv.size
    nk = r if kk is None else kk.size
    gU, SU = np.empty((nu, nk)), np.empty((nu, nk))
    gV, SV = np.empty((nv, nk)), np.empty((nv, nk))
    opt = lambda a: None if a is None else _ptr(a)
    rc = lib().nq_oracle_sign_grads_packed(_ptr(Uw), Uw.shape[1], _ptr(Vw), Vw.shape[1], _ptr(s1), _ptr(s2), d_out,
                                           d_in, r, _ptr(x), _ptr(yb), B, opt(ru), nu, opt(rv), nv, opt(kk), nk,
                                           _ptr(gU), _ptr(SU), _ptr(gV), _ptr(SV))
    if rc != 0:
        raise ValueError("nq_oracle_sign_grads_packed failed (%d)" % rc)
    return gU, SU, gV, SV


def double_to_f16(values) -> np.ndarray:
    """fp64 values -> fp16 bit patterns (round to nearest, ties to even)."""
    v = np.asarray(values, dtype=np.float64).ravel()
    return np.array([lib().nq_oracle_double_to_f16(float(a)) for a in v], dtype=np.uint16).reshape(np.shape(values))


def from_latent(Uh, Vh, ldu=None, ldv=None):
    """Balance the latent proxies (eta), extract the mean-absolute-value scales and pack the
    signs.  Returns (U words, V words, s1 fp16 bits, s2 fp16 bits, eta, s1 fp64, s2 fp64)."""
    Uh = _c(Uh, np.float32)
    Vh = _c(Vh, np.float32)
    d_out, r = Uh.shape
    d_in = Vh.shape[0]
    ldu = r // 32 if ldu is None else ldu
    ldv = r // 32 if ldv is None else ldv
    U = np.zeros((d_out, ldu), dtype=np.uint32)
    V = np.zeros((d_in, ldv), dtype=np.uint32)
    s1 = np.zeros(d_out, dtype=np.uint16)
    s2 = np.zeros(d_in, dtype=np.uint16)
    eta = np.zeros(1)
    s1d = np.zeros(d_out)
    s2d = np.zeros(d_in)
    rc = lib().nq_oracle_from_latent(_ptr(Uh), r, _ptr(Vh), r, d_out, d_in, r, _ptr(U), ldu, _ptr(V), ldv, _ptr(s1),
                                     _ptr(s2), _ptr(eta), _ptr(s1d), _ptr(s2d))
    if rc != 0:
        raise ValueError("nq_oracle_from_latent failed (%d)" % rc)
    return U, V, s1, s2, float(eta[0]), s1d, s2d


def factored_packed(Uw, Vw, s1_f16, s2_f16, r: int, x_bf16) -> np.ndarray:
    """y = s1 (.) (U (V^T (s2 (.) x))) in fp64 on the packed layout; [B][d_out]."""
    Uw = _c(Uw, np.uint32)
    Vw = _c(Vw, np.uint32)
    s1 = _c(s1_f16, np.uint16)
    s2 = _c(s2_f16, np.uint16)
    x = _c(np.atleast_2d(x_bf16), np.uint16)
    B = x.shape[0]
    y = np.empty((B, Uw.shape[0]), dtype=np.float64)
    rc = lib().nq_oracle_factored_packed(_ptr(Uw), Uw.shape[1], _ptr(Vw), Vw.shape[1], _ptr(s1), _ptr(s2),
                                         Uw.shape[0], Vw.shape[0], r, _ptr(x), B, _ptr(y))
    if rc != 0:
        raise ValueError("nq_oracle_factored_packed failed (%d)" % rc)
    return y


def silu_mul(g, u) -> np.ndarray:
    """h = bf16(silu(g) * u), silu(g) = g / (1 + exp(-g)), fp64 before the rounding."""
    g = _c(g, np.float64)
    u = _c(u, np.float64)
    h = np.empty(g.shape, dtype=np.uint16)
    lib().nq_oracle_silu_mul(_ptr(g), _ptr(u), g.size, _ptr(h))
    return h


def mlp(gate, up, down, x_bf16, rows=None, order="dense"):
    """Llama MLP block from three LRB projections, each given as (Uw, Vw, s1, s2, r).

    Not on the pages: the block that the 7B and 70B MLP workloads compose from three LRB
    layers (section 2 factorisation equation for each).  The gate and up projections are
    evaluated in fp64 and rounded to bf16 (the activation dtype), h = bf16(silu(g) * u), then
    the down projection is evaluated exactly on h.  ``order`` picks how gate and up are
    evaluated: "dense" is the definition (materialised W, exact up to the final fp64 sum);
    "factored" is s1 (.) (U (V^T (s2 (.) x))) in fp64, which is much faster at the 70B shapes
    and differs from the definition only by fp64 rounding (a bf16 rounding of g or u could
    differ only for a value within about 1e-15 of a midpoint).  ``rows`` selects output rows
    of the down projection.  Returns (y, S) of the down projection ([B][n_rows]) and h (bf16
    bits, [B][d_ff]).
    """
    if order == "dense":
        g, _ = dense_packed(*gate[:4], gate[4], x_bf16)
        u, _ = dense_packed(*up[:4], up[4], x_bf16)
    elif order == "factored":
        g = factored_packed(*gate[:4], gate[4], x_bf16)
        u = factored_packed(*up[:4], up[4], x_bf16)
    else:
        raise ValueError("order must be 'dense' or 'factored'")
    g16 = bf16_to_double(round_bf16(g))
    u16 = bf16_to_double(round_bf16(u))
    h = silu_mul(g16, u16)
    y, S = dense_packed(*down[:4], down[4], h, rows=rows)
    return y, S, h
