"""CPU oracle (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The library under
``verify_weight_streaming_b200`` never does, and the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, fp64), built into
``liboracle.so`` beside it; this module is the ctypes marshalling plus the
pass criteria written in terms of the oracle's outputs:

* matmul: ``|C_gpu - C64| <= 1e-5 * S`` per element, with ``S = sum |a*w|``;
  for a 16-bit output, half a unit of the output grid at ``|C64|`` is allowed on
  top (the unavoidable output rounding);
* top-k: indices equal to the oracle's top-k of the GPU's own fp32 logits,
  values bitwise equal to the logits at those indices.

Pins (what ties this oracle to the pages and to mathematics rather than to
itself) live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

F16, BF16 = 0, 1
FMT = {"f16": F16, "bf16": BF16}

REL_TOL = 1e-5   # |err| <= 1e-5 * sum|a*w|


def build(force: bool = False, src: str = SRC, out: str = LIB) -> str:
    """Compile oracle.c with gcc (-O2, no fast-math, no FMA contraction, OpenMP)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                        "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp, "-lm"],
                       check=True)
        os.replace(tmp, out)
    return out


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """ctypes view of one built copy of oracle.c (the tests also load mutants)."""

    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        L.oracle_dec_bf16.argtypes = [ctypes.c_uint16]
        L.oracle_dec_bf16.restype = ctypes.c_double
        L.oracle_dec_f16.argtypes = [ctypes.c_uint16]
        L.oracle_dec_f16.restype = ctypes.c_double
        L.oracle_matmul.argtypes = [P, I64, ctypes.c_int, P, I64, ctypes.c_int,
                                    I64, I64, I64, P, P, I64]
        L.oracle_matmul.restype = ctypes.c_int
        L.oracle_topk.argtypes = [P, I64, I64, I64, I32, P, P, I64]
        L.oracle_topk.restype = ctypes.c_int
        L.oracle_ulp_f16.argtypes = [ctypes.c_double]
        L.oracle_ulp_f16.restype = ctypes.c_double
        L.oracle_ulp_bf16.argtypes = [ctypes.c_double]
        L.oracle_ulp_bf16.restype = ctypes.c_double
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_cast_f32_bf16.argtypes = [P, I64, P, I64, I64, I64]
        L.oracle_sigmoid.argtypes = [ctypes.c_double]
        L.oracle_sigmoid.restype = ctypes.c_double
        self.L = L

    def dec_bf16(self, h: int) -> float:
        return self.L.oracle_dec_bf16(int(h) & 0xFFFF)

    def dec_f16(self, h: int) -> float:
        return self.L.oracle_dec_f16(int(h) & 0xFFFF)

    def matmul(self, a_bits: np.ndarray, a_fmt: str, wt_bits: np.ndarray, w_fmt: str):
        """(C64, S64) for C = A . W with W given k-contiguous as Wt[n][k]."""
        a = np.ascontiguousarray(a_bits, dtype=np.uint16)
        w = np.ascontiguousarray(wt_bits, dtype=np.uint16)
        if a.ndim != 2 or w.ndim != 2 or a.shape[1] != w.shape[1]:
            raise ValueError(f"shape mismatch {a.shape} x {w.shape}^T")
        m, k = a.shape
        n = w.shape[0]
        c = np.empty((m, n), dtype=np.float64)
        s = np.empty((m, n), dtype=np.float64)
        rc = self.L.oracle_matmul(_ptr(a), k, FMT[a_fmt], _ptr(w), k, FMT[w_fmt],
                                  m, n, k, _ptr(c), _ptr(s), n)
        if rc != 0:
            raise ValueError("oracle_matmul rejected its arguments")
        return c, s

    def topk(self, logits: np.ndarray, k: int):
        """(idx int32 [m,k], val fp32 [m,k]) by value desc, index asc, NaN first."""
        x = np.ascontiguousarray(logits, dtype=np.float32)
        if x.ndim != 2:
            raise ValueError("logits must be 2-D")
        m, n = x.shape
        idx = np.empty((m, k), dtype=np.int32)
        val = np.empty((m, k), dtype=np.float32)
        rc = self.L.oracle_topk(_ptr(x), n, m, n, k, _ptr(idx), _ptr(val), k)
        if rc != 0:
            raise ValueError("oracle_topk rejected its arguments")
        return idx, val

    def ulp(self, x, fmt: str) -> np.ndarray:
        f = self.L.oracle_ulp_f16 if fmt == "f16" else self.L.oracle_ulp_bf16
        flat = np.asarray(x, dtype=np.float64).ravel()
        return np.array([f(float(v)) for v in flat], dtype=np.float64).reshape(np.shape(x))

    def num_threads(self) -> int:
        return int(self.L.oracle_num_threads())

    def f32_to_bf16(self, x: float) -> int:
        return int(self.L.oracle_f32_to_bf16(float(x)))

    def cast_f32_bf16(self, x: np.ndarray) -> np.ndarray:
        """fp32 rows -> bf16 bit patterns (round to nearest even)."""
        x = np.ascontiguousarray(x, dtype=np.float32)
        rows, cols = x.shape
        y = np.empty((rows, cols), dtype=np.uint16)
        self.L.oracle_cast_f32_bf16(_ptr(x), cols, _ptr(y), cols, rows, cols)
        return y

    def sigmoid(self, x) -> np.ndarray:
        flat = np.asarray(x, dtype=np.float64).ravel()
        return np.array([self.L.oracle_sigmoid(float(v)) for v in flat]).reshape(np.shape(x))


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def dec_bf16(h: int) -> float:
    return default().dec_bf16(h)


def dec_f16(h: int) -> float:
    return default().dec_f16(h)


def matmul(a_bits, a_fmt, wt_bits, w_fmt):
    return default().matmul(a_bits, a_fmt, wt_bits, w_fmt)


def topk(logits, k):
    return default().topk(logits, k)


def ulp(x, fmt):
    return default().ulp(x, fmt)


def num_threads() -> int:
    return default().num_threads()


def cast_f32_bf16(x):
    return default().cast_f32_bf16(x)


def sigmoid(x):
    return default().sigmoid(x)


def gate_tolerance(c64: np.ndarray, s64: np.ndarray) -> np.ndarray:
    """Allowance for sigmoid(C): the GEMV's 1e-5*S through the sigmoid's
    slope (never above 1/4), plus 4 fp32 ulps of the result for the rounding of
    exp, the add and the divide."""
    sig = sigmoid(c64)
    return 0.25 * REL_TOL * s64 + 4.0 * np.spacing(np.abs(sig).astype(np.float32)).astype(np.float64)


def ulp_vec(x: np.ndarray, fmt: str) -> np.ndarray:
    """Vectorised twin of ``ulp`` (same definition), checked against it in the pins."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    frac_bits, min_exp = (10, -14) if fmt == "f16" else (7, -126)
    _, e = np.frexp(a)
    out = np.ldexp(1.0, (e - 1) - frac_bits)
    return np.where(a < np.ldexp(1.0, min_exp), np.ldexp(1.0, min_exp - frac_bits), out)


def tolerance(c64: np.ndarray, s64: np.ndarray, out_fmt: str = "f32") -> np.ndarray:
    """Per-element allowance: 1e-5*S, plus half an output ulp for 16-bit outputs."""
    tol = REL_TOL * s64
    if out_fmt in ("f16", "bf16"):
        tol = tol + 0.5 * ulp_vec(np.abs(c64) + tol, out_fmt)
    return tol


def check_matmul(c_gpu: np.ndarray, c64: np.ndarray, s64: np.ndarray, out_fmt: str = "f32"):
    """Returns (ok, worst_ratio, where) with ratio = |err| / tolerance."""
    err = np.abs(np.asarray(c_gpu, dtype=np.float64) - c64)
    tol = tolerance(c64, s64, out_fmt)
    # An exact zero allowance (all-zero row/col) must be met exactly.
    ratio = np.where(tol > 0, err / np.where(tol > 0, tol, 1.0), np.where(err > 0, np.inf, 0.0))
    if ratio.size == 0:
        return True, 0.0, None
    w = np.unravel_index(np.argmax(ratio), ratio.shape)
    return bool(ratio[w] <= 1.0), float(ratio[w]), tuple(int(v) for v in w)

