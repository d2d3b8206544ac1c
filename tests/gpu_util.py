"""Helpers for the GPU parity tests (tolerance, uploads).  Expected values always come
from the CPU oracle on the same seeded host inputs; nothing expected is taken from the GPU."""
import numpy as np
import pytest
import torch

# |y - y_ref| <= REL * S + ABS + ulp_bf16(y_ref) / 2 per output, with S = sum_j |W_ij x_j|
# (the magnitude of the terms of the oracle's own sum).  REL and ABS bound the arithmetic
# of the path; the half unit in the last place is the rounding of the result to the bf16
# output dtype, which alone reaches 2^-8 |y| and so exceeds REL * S whenever |y| is close to
# S (few terms, or terms of one sign).
REL = 2e-3
ABS = 1e-5


def half_ulp_bf16(v):
    """Half the spacing of bf16 numbers at |v| (8 significant bits; subnormal quantum 2^-133)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    _, e = np.frexp(a)  # a = m 2^e, 0.5 <= m < 1, so the bf16 spacing is 2^(e - 8)
    e = np.where(a == 0, -125, np.maximum(e, -125))
    return np.ldexp(0.5, e - 8)


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def nq():
    from rank_binary_factorized_b200 import nq as mod
    return mod


def upload_projection(p, device="cuda", ld_align_words=4):
    return nq().Layer.from_host(p.U, p.V, p.s1, p.s2, p.r, device=device, ld_align_words=ld_align_words)


def upload_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to("cuda").view(torch.bfloat16)


def download_bf16_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_bits_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# Headroom of every check_tolerance call in this process: (what, max err/tol with the
# bf16 half-ulp term, max err / (REL S + ABS) -- the stated bound without it).  Printed by
# the terminal summary hook in conftest.py and written as JSON to $NQ_MARGINS_JSON if set.
MARGINS = []


def check_tolerance(y_gpu_bits, y_ref, S, what=""):
    """Asserts the per-output bound and returns max(|err| / tol)."""
    y = bf16_bits_to_f64(y_gpu_bits)
    err = np.abs(y - y_ref)
    tol = REL * S + ABS + half_ulp_bf16(y_ref)
    ratio = err / tol
    strict = err / (REL * S + ABS)
    worst = np.unravel_index(np.argmax(ratio), ratio.shape)
    assert np.all(np.isfinite(y)), what + ": non-finite output"
    MARGINS.append((what, float(ratio.max()), float(strict.max())))
    assert ratio.max() <= 1.0, "%s: max err/tol %.3f at %s (y=%r ref=%r S=%r)" % (
        what, ratio.max(), worst, y[worst], y_ref[worst], S[worst])
    return float(ratio.max())
