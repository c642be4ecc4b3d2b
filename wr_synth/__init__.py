"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module only draws random numbers and names workload shapes. It holds none
of the method's arithmetic (no scales, codes, packing, rotation or contraction):
both sides receive the same fp32 weights, bf16 activations and sign bits from
here and do everything else themselves.

Distributions follow the workloads described on the pages and in the
configuration of this project: weights W ~ N(0, 0.02) in fp32, activations
x ~ N(0, 1) rounded to bf16, and a random sign vector for the block-128
random-sign Hadamard ("How do you fit a 4B LLM in 1.24 GB", Trick 1: a Hadamard
matrix "with random signs").

Weights are drawn in chunks of ``ROW_CHUNK`` rows, each chunk from its own
PCG64DXSM stream keyed by (seed, chunk index), so any row range can be
regenerated without drawing the rows before it.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

WEIGHT_STD = 0.02
ROW_CHUNK = 64

# One Qwen3-4B decoder layer (36 layers x 7 linears = 252 modules; "Qwen3-4B-Wringer-Q2.6",
# Recipe). (name, K = in_features, N = out_features, bits). v/up/down at 3 bits, the rest at
# 2 bits reproduces that page's code ledger of 2.520 bits per weight.
QWEN3_4B_LAYER = (
    ("q", 2560, 4096, 2),
    ("k", 2560, 1024, 2),
    ("v", 2560, 1024, 3),
    ("o", 4096, 2560, 2),
    ("gate", 2560, 9728, 2),
    ("up", 2560, 9728, 3),
    ("down", 9728, 2560, 3),
)
QWEN3_4B_LAYERS = 36


def module_seed(layer: int, index: int) -> int:
    """Seed of module ``index`` (0..6) of decoder layer ``layer``: 1000*layer + index."""
    return 1000 * layer + index


def _chunk_rng(seed: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64DXSM(np.random.SeedSequence([seed, chunk])))


def weights_fp32(seed: int, N: int, K: int, row0: int = 0, row1: int | None = None,
                 threads: int | None = None) -> np.ndarray:
    """Rows [row0, row1) of an N x K fp32 weight matrix with entries ~ N(0, WEIGHT_STD)."""
    if row1 is None:
        row1 = N
    assert 0 <= row0 <= row1 <= N
    out = np.empty((row1 - row0, K), dtype=np.float32)
    c0, c1 = row0 // ROW_CHUNK, (row1 + ROW_CHUNK - 1) // ROW_CHUNK

    def fill(c: int) -> None:
        lo, hi = c * ROW_CHUNK, min((c + 1) * ROW_CHUNK, N)
        block = _chunk_rng(seed, c).standard_normal((hi - lo, K), dtype=np.float32)
        block *= np.float32(WEIGHT_STD)
        a, b = max(lo, row0), min(hi, row1)
        out[a - row0:b - row0] = block[a - lo:b - lo]

    nthr = threads if threads is not None else min(32, os.cpu_count() or 1)
    if nthr <= 1 or c1 - c0 <= 1:
        for c in range(c0, c1):
            fill(c)
    else:
        with ThreadPoolExecutor(nthr) as ex:
            list(ex.map(fill, range(c0, c1)))
    return out


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); returns the uint16 bit patterns.
    Inputs are finite draws, so no NaN handling is needed."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def activations_bf16(seed: int, M: int, K: int) -> np.ndarray:
    """An M x K activation matrix x ~ N(0, 1), drawn in fp32 and rounded to bf16 (uint16 bits)."""
    rng = np.random.Generator(np.random.PCG64DXSM(np.random.SeedSequence([seed, 0x5A17])))
    return f32_to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32))


def sign_bits(seed: int, K: int) -> np.ndarray:
    """Random signs for the Hadamard rotation as a bitmask: bit k%32 of word k//32 set means -1."""
    rng = np.random.Generator(np.random.PCG64DXSM(np.random.SeedSequence([seed, 0x516E])))
    return rng.integers(0, 2**32, size=(K + 31) // 32, dtype=np.uint64).astype(np.uint32)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
