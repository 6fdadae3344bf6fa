"""Python binding of libmrgemm.so (ctypes; argument marshalling only).

Every function has the name of the C entry point it calls (see
``include/mrgemm.h``).  Tensors are torch CUDA tensors: torch supplies device
memory and the current stream, the library does all of the arithmetic.  16-bit
inputs may be ``torch.bfloat16`` / ``torch.float16`` or raw ``torch.int16``
patterns.  A status other than MR_OK raises ``MrError``.  If the compiled
library is missing the import fails: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

from ._build import LIB, build  # noqa: F401

MR_OK, MR_ERR_INVALID_ARG, MR_ERR_MISALIGNED, MR_ERR_UNSUPPORTED, MR_ERR_CUDA, MR_ERR_TIMEOUT = range(6)
MR_F16, MR_BF16, MR_F32 = 0, 1, 2
MR_GEMV_PDL = 0x1
MR_GEMV_SIGMOID = 0x2
MR_ROUTER_TWO_LAUNCH = 0x4
MR_DEVERR_GEMV_TIMEOUT, MR_DEVERR_GEMM_TIMEOUT, MR_DEVERR_TOPK_TIMEOUT, MR_DEVERR_SELFTEST = 1, 2, 4, 8

EXPORTS = (
    "mrgemv_bf16", "mrgemv_bf16_ex", "mrgemv_bf16_plan", "router_topk", "router_topk_ex",
    "router_topk_merge", "router_gemv_topk",
    "router_gemv_topk_workspace_bytes", "router_gemv_topk_noalloc", "router_gemv_topk_noalloc_max_logits", "gemm_f16_grouped",
    "gemm_f16_grouped_select_tile", "cast_f32_bf16", "gemm_f16_ex", "gemm_f16", "gemm_f16_num_tiles",
    "gemm_f16_tile_name", "gemm_f16_select_tile", "mr_poll_errors", "mr_selftest_wait_timeout",
    "mr_status_str", "mr_version",
)


class MrError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call}: {status_str(status)}")


def _load() -> ctypes.CDLL:
    from . import _build
    if _build.stale():
        # Sources newer than the library (or no library): compile it now with
        # nvcc.  Without a toolkit this raises; there is no fallback path.
        try:
            _build.build()
        except Exception as exc:
            raise ImportError(f"{LIB} is missing or stale and could not be built: {exc}") from exc
    L = ctypes.CDLL(LIB)
    P, I64, I32, U32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32
    L.mrgemv_bf16.argtypes = [P, I64, P, I64, P, I64, I32, I32, I32, P]
    L.mrgemv_bf16_ex.argtypes = [P, I64, P, I64, P, I64, I32, I32, I32, U32, P]
    L.mrgemv_bf16_plan.argtypes = [I32, I32, I32, U32, I32, I32, P]
    L.router_topk.argtypes = [P, I64, I32, I32, I32, P, P, I64, P]
    L.router_topk_ex.argtypes = [P, I64, I32, I32, I32, P, P, I64, I32, P]
    L.router_topk_merge.argtypes = [P, P, I32, I32, I32, I64, I64, I32, P, P, I64, P]
    L.router_gemv_topk.argtypes = [P, I64, P, I64, P, I64, I32, I32, I32, I32, P, P, I64, P,
                                   ctypes.c_size_t, U32, P]
    L.router_gemv_topk_workspace_bytes.argtypes = [I32, I32, I32]
    L.router_gemv_topk_workspace_bytes.restype = ctypes.c_size_t
    L.router_gemv_topk_noalloc.argtypes = [P, I64, P, I64, P, I64, I32, I32, I32, I32, P, P, I64, U32, P]
    L.router_gemv_topk_noalloc_max_logits.argtypes = []
    L.router_gemv_topk_noalloc_max_logits.restype = ctypes.c_size_t
    L.gemm_f16.argtypes = [P, I64, P, I64, P, I64, I32, I32, I32, I32, I32, I32, P]
    L.gemm_f16_grouped.argtypes = [P, I64, P, I64, P, I64, I32, I32, I32, I32, I32, I32, I32, P]
    L.gemm_f16_grouped_select_tile.argtypes = [I32, I32, I32, I32]
    L.cast_f32_bf16.argtypes = [P, I64, P, I64, I32, I32, P]
    L.gemm_f16_ex.argtypes = [P, I64, P, I64, P, I64, I32, I32, I32, I32, I32, I32, I32, P]
    L.gemm_f16_num_tiles.argtypes = []
    L.gemm_f16_tile_name.argtypes = [I32]
    L.gemm_f16_tile_name.restype = ctypes.c_char_p
    L.gemm_f16_select_tile.argtypes = [I32, I32, I32]
    L.mr_poll_errors.argtypes = [P, ctypes.POINTER(U32)]
    L.mr_selftest_wait_timeout.argtypes = [I32, P]
    L.mr_status_str.argtypes = [ctypes.c_int]
    L.mr_status_str.restype = ctypes.c_char_p
    L.mr_version.argtypes = []
    L.mr_version.restype = ctypes.c_char_p
    for name in ("mrgemv_bf16", "mrgemv_bf16_ex", "mrgemv_bf16_plan", "router_topk", "router_topk_ex",
                 "router_topk_merge", "router_gemv_topk",
                 "router_gemv_topk_noalloc", "gemm_f16_grouped", "gemm_f16_grouped_select_tile",
                 "cast_f32_bf16", "gemm_f16_ex", "gemm_f16", "gemm_f16_num_tiles",
                 "gemm_f16_select_tile", "mr_poll_errors", "mr_selftest_wait_timeout"):
        getattr(L, name).restype = ctypes.c_int
    return L


lib = _load()


def status_str(status: int) -> str:
    return lib.mr_status_str(int(status)).decode()


def version() -> str:
    return lib.mr_version().decode()


def _check(status: int, call: str) -> None:
    if status != MR_OK:
        raise MrError(status, call)


_current_raw_stream = None


def _current_stream_handle() -> int:
    """The current CUDA stream of the current device, as torch sees it."""
    global _current_raw_stream
    if _current_raw_stream is None:
        import torch
        raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
        dev = getattr(torch._C, "_cuda_getDevice", None)
        if raw is not None and dev is not None:
            _current_raw_stream = lambda: raw(dev())  # noqa: E731  (one C++ call each, per launch)
        else:
            _current_raw_stream = lambda: torch.cuda.current_stream().cuda_stream  # noqa: E731
    return _current_raw_stream()


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(_current_stream_handle())
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _rows(t, name):
    st = t.stride()
    if len(st) != 2 or st[1] != 1:
        raise ValueError(f"{name} must be a 2-D tensor with unit column stride")
    sh = t.shape
    return sh[0], sh[1], st[0]


def _dtype_code(t) -> int:
    import torch
    return {torch.float16: MR_F16, torch.bfloat16: MR_BF16, torch.float32: MR_F32,
            torch.int16: MR_BF16}.get(t.dtype, -1)


def mrgemv_bf16(A, Wt, C, stream=None, flags: int = 0) -> None:
    """C[m,n] (fp32) = A[m,k] (bf16) . Wt[n,k]^T (bf16); m <= 16."""
    m, k, lda = _rows(A, "A")
    n, kw, ldw = _rows(Wt, "Wt")
    mc, nc, ldc = _rows(C, "C")
    if kw != k or mc != m or nc != n:
        raise ValueError(f"shape mismatch A{tuple(A.shape)} Wt{tuple(Wt.shape)} C{tuple(C.shape)}")
    st = lib.mrgemv_bf16_ex(A.data_ptr(), lda, Wt.data_ptr(), ldw, C.data_ptr(), ldc,
                            m, n, k, flags, _stream(stream))
    _check(st, "mrgemv_bf16")


PLAN_FIELDS = ("grid", "threads", "smem_bytes", "ring_slots", "k_warps", "column_warps",
               "row_bucket", "columns_per_group")


def mrgemv_bf16_plan(m: int, n: int, k: int, flags: int, sm_count: int, smem_optin: int) -> dict:
    """The launch plan of mrgemv_bf16_ex for these sizes on a described device."""
    out = (ctypes.c_int32 * 8)()
    _check(lib.mrgemv_bf16_plan(m, n, k, flags, sm_count, smem_optin, out), "mrgemv_bf16_plan")
    return dict(zip(PLAN_FIELDS, list(out)))


def router_topk(logits, topk: int, idx, val=None, stream=None) -> None:
    """idx[m,topk] (int32), val[m,topk] (fp32, optional) = per-row top-k of logits[m,n]."""
    m, n, ldl = _rows(logits, "logits")
    mi, ki, ldo = _rows(idx, "idx")
    if mi != m or ki < topk:
        raise ValueError("idx shape mismatch")
    vptr = None
    if val is not None:
        mv, kv, ldv = _rows(val, "val")
        if mv != m or kv < topk or ldv != ldo:
            raise ValueError("val must match idx's shape and stride")
        vptr = val.data_ptr()
    st = lib.router_topk(logits.data_ptr(), ldl, m, n, topk, idx.data_ptr(), vptr, ldo, _stream(stream))
    _check(st, "router_topk")


def router_topk_ex(logits, topk: int, idx, val=None, index_base: int = 0, stream=None) -> None:
    """router_topk of a shard of columns: indices are written as index_base + column."""
    m, n, ldl = _rows(logits, "logits")
    mi, ki, ldo = _rows(idx, "idx")
    if mi != m or ki < topk:
        raise ValueError("idx shape mismatch")
    vptr = None
    if val is not None:
        mv, kv, ldv = _rows(val, "val")
        if mv != m or kv < topk or ldv != ldo:
            raise ValueError("val must match idx's shape and stride")
        vptr = val.data_ptr()
    st = lib.router_topk_ex(logits.data_ptr(), ldl, m, n, topk, idx.data_ptr(), vptr, ldo, index_base,
                            _stream(stream))
    _check(st, "router_topk_ex")


def router_topk_merge(cand_val, cand_idx, topk: int, idx, val=None, stream=None) -> None:
    """Per-row top-k of candidate lists laid out [groups, m, per_group] (fp32
    values, int32 global indices, -1 = empty), e.g. an all-gather of every
    shard's router_topk_ex output."""
    if cand_val.dim() != 3 or tuple(cand_idx.shape) != tuple(cand_val.shape):
        raise ValueError("cand_val and cand_idx must be [groups, m, per_group] of the same shape")
    if cand_val.stride() != cand_idx.stride() or cand_val.stride(2) != 1:
        raise ValueError("candidates need a common layout with unit stride in the last dimension")
    groups, m, per = cand_val.shape
    mi, ki, ldo = _rows(idx, "idx")
    if mi != m or ki < topk:
        raise ValueError("idx shape mismatch")
    vptr = None
    if val is not None:
        mv, kv, ldv = _rows(val, "val")
        if mv != m or kv < topk or ldv != ldo:
            raise ValueError("val must match idx's shape and stride")
        vptr = val.data_ptr()
    st = lib.router_topk_merge(cand_val.data_ptr(), cand_idx.data_ptr(), m, groups, per, cand_val.stride(1),
                               cand_val.stride(0), topk, idx.data_ptr(), vptr, ldo, _stream(stream))
    _check(st, "router_topk_merge")


MR_ROUTER_TICKET_BYTES = 256


def router_gemv_topk_workspace_bytes(m: int, n: int, logits_provided: bool) -> int:
    return int(lib.router_gemv_topk_workspace_bytes(m, n, 1 if logits_provided else 0))


def router_gemv_topk(A, Wt, topk: int, idx, val=None, logits=None, workspace=None, stream=None,
                     flags: int = 0) -> None:
    """GEMV + per-row top-k in one launch (or, with MR_ROUTER_TWO_LAUNCH, the
    GEMV kernel then the top-k kernel).  ``workspace``: a zeroed CUDA tensor
    of at least router_gemv_topk_workspace_bytes(...) bytes (each fused call
    leaves its tag array zero again)."""
    m, k, lda = _rows(A, "A")
    n, kw, ldw = _rows(Wt, "Wt")
    if kw != k:
        raise ValueError("A and Wt disagree on k")
    mi, ki, ldo = _rows(idx, "idx")
    if mi != m or ki < topk:
        raise ValueError("idx shape mismatch")
    lptr, ldl = None, n
    if logits is not None:
        ml, nl, ldl = _rows(logits, "logits")
        if ml != m or nl != n:
            raise ValueError("logits shape mismatch")
        lptr = logits.data_ptr()
    vptr = None
    if val is not None:
        mv, kv, ldv = _rows(val, "val")
        if mv != m or kv < topk or ldv != ldo:
            raise ValueError("val must match idx's shape and stride")
        vptr = val.data_ptr()
    if workspace is None:
        raise ValueError("router_gemv_topk needs a zero-initialised workspace tensor")
    wbytes = workspace.numel() * workspace.element_size()
    st = lib.router_gemv_topk(A.data_ptr(), lda, Wt.data_ptr(), ldw, lptr, ldl, m, n, k, topk,
                              idx.data_ptr(), vptr, ldo, workspace.data_ptr(), wbytes, flags,
                              _stream(stream))
    _check(st, "router_gemv_topk")


def gemm_f16(A, Wt, C, tile_id: int = -1, in_dtype: int | None = None, stream=None, raster: int = 0) -> None:
    """C[M,N] = A[M,K] . Wt[N,K]^T on tcgen05; dtypes from the tensors (int16 = bf16 bits)."""
    M, K, lda = _rows(A, "A")
    N, kw, ldw = _rows(Wt, "Wt")
    mc, nc, ldc = _rows(C, "C")
    if kw != K or mc != M or nc != N:
        raise ValueError("shape mismatch")
    idt = _dtype_code(A) if in_dtype is None else in_dtype
    st = lib.gemm_f16_ex(A.data_ptr(), lda, Wt.data_ptr(), ldw, C.data_ptr(), ldc, M, N, K,
                         idt, _dtype_code(C), tile_id, raster, _stream(stream))
    _check(st, "gemm_f16")


def gemm_f16_grouped(A, Wts, Cs, tile_id: int = -1, in_dtype: int | None = None, stream=None) -> None:
    """Cs[g] = A . Wts[g]^T for every g in one launch (lists of equal-shape tensors)."""
    M, K, lda = _rows(A, "A")
    if len(Wts) != len(Cs) or not Wts:
        raise ValueError("Wts and Cs must be non-empty lists of the same length")
    N, kw, ldw = _rows(Wts[0], "Wts[0]")
    _, _, ldc = _rows(Cs[0], "Cs[0]")
    for w, c in zip(Wts, Cs):
        if tuple(w.shape) != (N, K) or w.stride(0) != ldw or tuple(c.shape) != (M, N) or c.stride(0) != ldc:
            raise ValueError("every Wts[g] must be [N,K] and every Cs[g] [M,N] with common strides")
    G = len(Wts)
    wp = (ctypes.c_void_p * G)(*[w.data_ptr() for w in Wts])
    cp = (ctypes.c_void_p * G)(*[c.data_ptr() for c in Cs])
    idt = _dtype_code(A) if in_dtype is None else in_dtype
    st = lib.gemm_f16_grouped(A.data_ptr(), lda, wp, ldw, cp, ldc, M, N, K, G, idt, _dtype_code(Cs[0]),
                              tile_id, _stream(stream))
    _check(st, "gemm_f16_grouped")


def gemm_f16_grouped_select_tile(M: int, N: int, K: int, G: int) -> int:
    return int(lib.gemm_f16_grouped_select_tile(M, N, K, G))


def cast_f32_bf16(X, Y, stream=None) -> None:
    """Y (bf16 or int16 bits) = X (fp32) rounded to nearest even."""
    rows, cols, ldx = _rows(X, "X")
    ry, cy, ldy = _rows(Y, "Y")
    if (ry, cy) != (rows, cols):
        raise ValueError("X and Y shapes differ")
    _check(lib.cast_f32_bf16(X.data_ptr(), ldx, Y.data_ptr(), ldy, rows, cols, _stream(stream)), "cast_f32_bf16")


def gemm_f16_num_tiles() -> int:
    return int(lib.gemm_f16_num_tiles())


def gemm_f16_tile_name(tile_id: int):
    r = lib.gemm_f16_tile_name(tile_id)
    return None if r is None else r.decode()


def gemm_f16_select_tile(M: int, N: int, K: int) -> int:
    return int(lib.gemm_f16_select_tile(M, N, K))


def mr_poll_errors(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error bits."""
    flags = ctypes.c_uint32(0)
    st = lib.mr_poll_errors(_stream(stream), ctypes.byref(flags))
    if st not in (MR_OK, MR_ERR_TIMEOUT):
        raise MrError(st, "mr_poll_errors")
    return int(flags.value)


def mr_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    _check(lib.mr_selftest_wait_timeout(limit_us, _stream(stream)), "mr_selftest_wait_timeout")
