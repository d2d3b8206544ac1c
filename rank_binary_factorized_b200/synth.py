"""Seeded synthetic inputs for the low-rank binary (LRB) layers.

This module only draws random numbers and lays them out; it holds none of the method's
arithmetic.  The CUDA path and the CPU oracle both take their inputs from here, so the two
sides see the same bits.

Recipe (one per projection, all from ``numpy.random.default_rng``):

* signs: iid +-1 with p = 1/2, drawn directly as uniform random uint32 words (every bit an
  independent fair coin), 32 signs per word along r, bit 1 for +1; pad words (ld > r/32) 0;
* scales s1, s2: fp16(0.02 * |N(0, 1)|), round to nearest even;
* activations x: bf16(N(0, 1)), round to nearest even;
* latent factors for the pack step: fp32 N(0, 1).

Workloads are the Llama-2 shapes the method is quoted on (d_out, d_in, r per projection).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

BASE_SEED = 20260206


@dataclass
class Projection:
    """One LRB linear layer, as host arrays in the packed layout.

    U: uint32 [d_out][ldu]; V: uint32 [d_in][ldv]; s1: fp16 bits [d_out]; s2: fp16 bits [d_in].
    """

    name: str
    d_out: int
    d_in: int
    r: int
    U: np.ndarray
    V: np.ndarray
    s1: np.ndarray
    s2: np.ndarray

    @property
    def ldu(self) -> int:
        return int(self.U.shape[1])

    @property
    def ldv(self) -> int:
        return int(self.V.shape[1])

    def packed_bytes(self) -> int:
        return 4 * (self.d_out * self.r // 32 + self.d_in * self.r // 32)

    def scale_bytes(self) -> int:
        return 2 * (self.d_out + self.d_in)


# name -> list of (projection name, d_out, d_in, r)
WORKLOADS = {
    "tiny": [("proj", 256, 512, 128)],
    "attn7b": [("proj", 4096, 4096, 2048)],
    "mlp7b": [("gate", 11008, 4096, 2368), ("up", 11008, 4096, 2368), ("down", 4096, 11008, 2368)],
    "layer70b": [
        ("q", 8192, 8192, 2240),
        ("k", 1024, 8192, 512),
        ("v", 1024, 8192, 512),
        ("o", 8192, 8192, 2240),
        ("gate", 28672, 8192, 3520),
        ("up", 28672, 8192, 3520),
        ("down", 8192, 28672, 3520),
    ],
    "prefill70b": [("gate", 28672, 8192, 3520)],
}

# Seed offsets per workload (base seed + index in this order).
_ORDER = ["tiny", "attn7b", "mlp7b", "layer70b", "prefill70b"]


def workload_seed(workload: str) -> int:
    return BASE_SEED + _ORDER.index(workload)


def rng_for(seed: int, *keys: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, *keys]))


def sign_words(rng: np.random.Generator, rows: int, r: int, ld: int | None = None) -> np.ndarray:
    """iid fair sign bits as uint32 words [rows][ld]; words past r/32 are 0."""
    if r % 32 != 0:
        raise ValueError("r must be a multiple of 32")
    ld = r // 32 if ld is None else ld
    out = np.zeros((rows, ld), dtype=np.uint32)
    out[:, : r // 32] = rng.integers(0, 2**32, size=(rows, r // 32), dtype=np.uint64).astype(np.uint32)
    return out


def scales_f16(rng: np.random.Generator, n: int, scale: float = 0.02) -> np.ndarray:
    """fp16(scale * |N(0,1)|) as uint16 bit patterns."""
    return (scale * np.abs(rng.standard_normal(n))).astype(np.float16).view(np.uint16)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bfloat16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def acts_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    """bf16(N(0,1)) bit patterns."""
    return f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def latent_f32(rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    return rng.standard_normal((rows, cols)).astype(np.float32)


def make_projection(name: str, d_out: int, d_in: int, r: int, seed: int, key: int = 0,
                    ldu: int | None = None, ldv: int | None = None) -> Projection:
    rng = rng_for(seed, key)
    U = sign_words(rng, d_out, r, ldu)
    V = sign_words(rng, d_in, r, ldv)
    s1 = scales_f16(rng, d_out)
    s2 = scales_f16(rng, d_in)
    return Projection(name, d_out, d_in, r, U, V, s1, s2)


def make_workload(workload: str, instance: int = 0) -> list[Projection]:
    """All projections of a named workload; ``instance`` gives distinct weight copies."""
    seed = workload_seed(workload)
    return [make_projection(n, do, di, r, seed, key=1000 * instance + idx)
            for idx, (n, do, di, r) in enumerate(WORKLOADS[workload])]


def make_input(workload: str, d_in: int, batch: int, key: int = 0) -> np.ndarray:
    """bf16 activations [batch][d_in] for a workload."""
    return acts_bf16(rng_for(workload_seed(workload), 7_000_000 + key), (batch, d_in))
