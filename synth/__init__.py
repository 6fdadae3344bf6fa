"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only *draws numbers*: it holds none of the matmul, reduction or
selection arithmetic that the library computes, so the CPU oracle and the CUDA
path can both consume its output without sharing any of the method's code.

Generator (one fixed reading, applied everywhere):

* splitmix64, counter based: draw ``i`` of a stream with seed ``s`` is
  ``mix(s + (i + 1) * 0x9E3779B97F4A7C15 mod 2**64)`` with the usual
  splitmix64 finaliser (shifts 30/27/31, multipliers 0xBF58476D1CE4E5B9 and
  0x94D049BB133111EB).
* Uniforms: ``u = ((z >> 11) + 1) * 2**-53`` lies in (0, 1].
* Normals: Box-Muller in fp64 on consecutive pairs of draws,
  ``n[2j] = r cos t`` and ``n[2j+1] = r sin t`` with ``r = sqrt(-2 ln u[2j])``
  and ``t = 2 pi u[2j+1]``.
* ``N(mu, s)`` means mean ``mu`` and *standard deviation* ``s``
  (so ``W ~ N(0, 1/sqrt(k))`` gives outputs of unit standard deviation).
* Values are scaled in fp64, rounded to fp32 (round to nearest even), then to
  bf16 or f16 (round to nearest even).  The 16-bit patterns are the inputs;
  both sides decode the same bits.
* Seeds: ``0x5EED0000 + 16 * workload + stream``; stream 0 is A, stream
  ``1 + w`` is the w-th weight matrix of the workload.

Workloads follow the shapes named on the pages: the Qwen FFN inner dim k=896
of the nx_batchscale_kat.nx note, the 2.6 MB router (2560 x 512) of Strata
PR #109 ("What", router bullet), and the Walbe / big-N prompt-chunk GEMMs of
the "opus r35 track A" audit (section 2, gemm_f16 tiles).
"""
from __future__ import annotations

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

SEED_BASE = 0x5EED0000

# Workload ids used in seeds (one per synthetic workload family).
WL_GEMV_FFN = 0      # A[m,896] x W[896,4864] bf16
WL_ROUTER = 1        # A[m,2560] x W_r[2560,512] bf16 + top-10
WL_NARROW = 2        # A[M,2560] x 36 x W[2560,96] f16
WL_CHUNK = 3         # A[M,2560] x W[2560,N] f16
WL_SWEEP = 4         # m-sweep, bf16


def seed_for(workload: int, stream: int) -> int:
    return (SEED_BASE + 16 * int(workload) + int(stream)) & 0xFFFFFFFFFFFFFFFF


def splitmix64(seed: int, count: int, start: int = 0) -> np.ndarray:
    """Draws ``start .. start+count-1`` of the counter-based splitmix64 stream."""
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        z = np.uint64(seed) + i * GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform01(seed: int, count: int) -> np.ndarray:
    z = splitmix64(seed, count)
    return ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def normal(seed: int, count: int, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """``count`` fp64 normals by Box-Muller on consecutive uniform pairs."""
    pairs = (count + 1) // 2
    u = uniform01(seed, 2 * pairs)
    r = np.sqrt(-2.0 * np.log(u[0::2]))
    t = (2.0 * np.pi) * u[1::2]
    out = np.empty(2 * pairs, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out[:count] * std + mean


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))
    return ((b + bias) >> np.uint64(16)).astype(np.uint16)


def to_bits(x64: np.ndarray, fmt: str) -> np.ndarray:
    """fp64 values -> fp32 (RNE) -> 16-bit pattern of ``fmt`` ('bf16' or 'f16')."""
    x32 = np.asarray(x64, dtype=np.float64).astype(np.float32)
    if fmt == "bf16":
        return f32_to_bf16_bits(x32)
    if fmt == "f16":
        return x32.astype(np.float16).view(np.uint16)
    raise ValueError(f"unknown 16-bit format {fmt!r}")


def normal_bits(seed: int, shape, fmt: str, std: float, mean: float = 0.0) -> np.ndarray:
    """A seeded ``shape`` array of ``fmt`` bit patterns drawn from N(mean, std)."""
    count = int(np.prod(shape))
    return to_bits(normal(seed, count, mean, std), fmt).reshape(shape)


def bits_to_float32(bits: np.ndarray, fmt: str) -> np.ndarray:
    """Reinterpret 16-bit patterns as fp32 values (for torch upload and plots)."""
    bits = np.asarray(bits, dtype=np.uint16)
    if fmt == "bf16":
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    if fmt == "f16":
        return bits.view(np.float16).astype(np.float32)
    raise ValueError(fmt)


def integer_bits(seed: int, shape, fmt: str, lo: int, hi: int) -> np.ndarray:
    """Small integers in [lo, hi], exactly representable in bf16 and f16 (|v| <= 256)."""
    count = int(np.prod(shape))
    z = splitmix64(seed, count)
    span = np.uint64(hi - lo + 1)
    v = (z % span).astype(np.int64) + lo
    return to_bits(v.astype(np.float64), fmt).reshape(shape)


def choice_bits(seed: int, shape, fmt: str, values) -> np.ndarray:
    """Values drawn uniformly from a small list (tie-heavy rows for top-k)."""
    values = np.asarray(values, dtype=np.float64)
    count = int(np.prod(shape))
    z = splitmix64(seed, count)
    v = values[(z % np.uint64(len(values))).astype(np.int64)]
    return to_bits(v, fmt).reshape(shape)


def choice_f32(seed: int, shape, values) -> np.ndarray:
    values = np.asarray(values, dtype=np.float32)
    count = int(np.prod(shape))
    z = splitmix64(seed, count)
    return values[(z % np.uint64(len(values))).astype(np.int64)].reshape(shape)


# --- workload recipes -------------------------------------------------------

def gemv_ffn(m: int, k: int = 896, n: int = 4864, w_index: int = 0):
    """A[m,k] bf16 ~ N(0,1); W_t[n,k] bf16 ~ N(0, 1/sqrt(k))."""
    a = normal_bits(seed_for(WL_GEMV_FFN, 0), (m, k), "bf16", 1.0)
    w = normal_bits(seed_for(WL_GEMV_FFN, 1 + w_index), (n, k), "bf16", 1.0 / np.sqrt(k))
    return a, w


def router(m: int, k: int = 2560, n: int = 512, w_index: int = 0):
    """A[m,k] bf16 ~ N(0,1); W_r stored as W_t[n,k] bf16 ~ N(0, 0.02)."""
    a = normal_bits(seed_for(WL_ROUTER, 0), (m, k), "bf16", 1.0)
    w = normal_bits(seed_for(WL_ROUTER, 1 + w_index), (n, k), "bf16", 0.02)
    return a, w


def narrow(M: int, k: int = 2560, n: int = 96, w_index: int = 0, fmt: str = "f16"):
    """A[M,k] ~ N(0,1); the w_index-th of 36 W_t[96,k] ~ N(0, 1/sqrt(k))."""
    a = normal_bits(seed_for(WL_NARROW, 0), (M, k), fmt, 1.0)
    w = normal_bits(seed_for(WL_NARROW, 1 + w_index), (n, k), fmt, 1.0 / np.sqrt(k))
    return a, w


def chunk(M: int, N: int, k: int = 2560, fmt: str = "f16"):
    """A[M,k] ~ N(0,1); W_t[N,k] ~ N(0, 1/sqrt(k)) (every N takes a prefix of stream 1)."""
    a = normal_bits(seed_for(WL_CHUNK, 0), (M, k), fmt, 1.0)
    w = normal_bits(seed_for(WL_CHUNK, 1), (N, k), fmt, 1.0 / np.sqrt(k))
    return a, w
