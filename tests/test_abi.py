"""The C ABI on a machine without a GPU: exports, validation, status codes.

Only host-side validation runs here; every call below returns before any CUDA
call is made, except the one that checks a valid call reports MR_ERR_CUDA
when no device exists.
"""
import ctypes
import os
import re

import pytest

import verify_weight_streaming_b200 as mr

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "mrgemm.h")
P = ctypes.c_void_p
A16 = P(256)            # 16-byte aligned stand-in pointers (never dereferenced)
BAD = P(258)            # 2-byte aligned


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_0-9]+)\s*\(", text)) - {"defined"})


def test_header_declares_and_library_exports_every_entry_point():
    names = declared_functions()
    assert set(mr.EXPORTS) <= set(names), set(mr.EXPORTS) - set(names)
    for name in names:
        assert hasattr(mr.lib, name), f"libmrgemm.so does not export {name}"


def test_status_strings():
    for code, name in enumerate(["MR_OK", "MR_ERR_INVALID_ARG", "MR_ERR_MISALIGNED",
                                 "MR_ERR_UNSUPPORTED", "MR_ERR_CUDA", "MR_ERR_TIMEOUT"]):
        assert mr.status_str(code) == name
    assert mr.status_str(99) == "MR_ERR_UNKNOWN"
    assert "sm_100a" in mr.version()


def gemv(A=A16, lda=64, W=A16, ldw=64, C=A16, ldc=32, m=4, n=32, k=64, flags=0):
    return mr.lib.mrgemv_bf16_ex(A, lda, W, ldw, C, ldc, m, n, k, flags, None)


@pytest.mark.parametrize("kw,code", [
    (dict(A=None), mr.MR_ERR_INVALID_ARG), (dict(W=None), mr.MR_ERR_INVALID_ARG),
    (dict(C=None), mr.MR_ERR_INVALID_ARG), (dict(m=0), mr.MR_ERR_INVALID_ARG),
    (dict(n=0), mr.MR_ERR_INVALID_ARG), (dict(k=0), mr.MR_ERR_INVALID_ARG),
    (dict(lda=56), mr.MR_ERR_INVALID_ARG), (dict(ldc=31), mr.MR_ERR_INVALID_ARG),
    (dict(flags=4), mr.MR_ERR_INVALID_ARG),
    (dict(k=60, lda=64, ldw=64), mr.MR_ERR_MISALIGNED), (dict(lda=68), mr.MR_ERR_MISALIGNED),
    (dict(A=BAD), mr.MR_ERR_MISALIGNED), (dict(W=BAD), mr.MR_ERR_MISALIGNED),
    (dict(m=17), mr.MR_ERR_UNSUPPORTED),
])
def test_gemv_validation(kw, code):
    assert gemv(**kw) == code


def test_gemv_valid_call_without_device_is_a_cuda_error():
    assert gemv() == mr.MR_ERR_CUDA


def topk(logits=A16, ldl=512, m=4, n=512, k=10, idx=A16, val=None, ldo=10):
    return mr.lib.router_topk(logits, ldl, m, n, k, idx, val, ldo, None)


@pytest.mark.parametrize("kw,code", [
    (dict(logits=None), mr.MR_ERR_INVALID_ARG), (dict(idx=None), mr.MR_ERR_INVALID_ARG),
    (dict(m=0), mr.MR_ERR_INVALID_ARG), (dict(n=0), mr.MR_ERR_INVALID_ARG),
    (dict(k=0), mr.MR_ERR_INVALID_ARG), (dict(n=8, ldl=8, k=9, ldo=9), mr.MR_ERR_INVALID_ARG),
    (dict(ldl=500), mr.MR_ERR_INVALID_ARG), (dict(ldo=9), mr.MR_ERR_INVALID_ARG),
    (dict(k=33, ldo=33), mr.MR_ERR_UNSUPPORTED), (dict(logits=P(258)), mr.MR_ERR_MISALIGNED),
])
def test_topk_validation(kw, code):
    assert topk(**kw) == code


def test_selftest_limits():
    assert mr.lib.mr_selftest_wait_timeout(0, None) == mr.MR_ERR_INVALID_ARG
    assert mr.lib.mr_selftest_wait_timeout(1000001, None) == mr.MR_ERR_INVALID_ARG


def gemm(A=A16, lda=64, W=A16, ldw=64, C=A16, ldc=32, M=4, N=32, K=64, ind=mr.MR_F16, outd=mr.MR_F16, tile=-1):
    return mr.lib.gemm_f16(A, lda, W, ldw, C, ldc, M, N, K, ind, outd, tile, None)


@pytest.mark.parametrize("kw,code", [
    (dict(A=None), mr.MR_ERR_INVALID_ARG), (dict(W=None), mr.MR_ERR_INVALID_ARG),
    (dict(C=None), mr.MR_ERR_INVALID_ARG), (dict(M=0), mr.MR_ERR_INVALID_ARG),
    (dict(N=0), mr.MR_ERR_INVALID_ARG), (dict(K=0), mr.MR_ERR_INVALID_ARG),
    (dict(lda=56), mr.MR_ERR_INVALID_ARG), (dict(ldc=24), mr.MR_ERR_INVALID_ARG),
    (dict(ind=mr.MR_F32), mr.MR_ERR_INVALID_ARG), (dict(outd=7), mr.MR_ERR_INVALID_ARG),
    (dict(tile=12), mr.MR_ERR_INVALID_ARG), (dict(tile=-2), mr.MR_ERR_INVALID_ARG),
    (dict(K=60, lda=64, ldw=64), mr.MR_ERR_MISALIGNED), (dict(ldc=36), mr.MR_ERR_MISALIGNED),
    (dict(C=P(264)), mr.MR_ERR_MISALIGNED), (dict(A=BAD), mr.MR_ERR_MISALIGNED),
])
def test_gemm_validation(kw, code):
    assert gemm(**kw) == code


def test_gemm_tiles_and_selector_on_host():
    n = mr.gemm_f16_num_tiles()
    assert n == 12
    names = [mr.gemm_f16_tile_name(t) for t in range(n)]
    assert names == ["128x32", "128x64", "128x96", "128x128", "128x192", "128x256", "64x128", "64x256",
                     "256x256", "256x128", "64x32", "64x64"]
    assert mr.gemm_f16_tile_name(n) is None and mr.gemm_f16_tile_name(-1) is None
    assert mr.gemm_f16_select_tile(0, 96, 2560) == -1
    for M in (1, 150, 306, 1983, 2048):
        for N in (1, 96, 512, 6144):
            assert 0 <= mr.gemm_f16_select_tile(M, N, 2560) < n


def test_selector_tail_rule_and_measured_choices():
    """Row tails count as whole tiles (64 or 128 rows): every M in the same
    64-row band (the same number of 64-row and of 128-row tiles) gets the
    same tile.  And on shapes where one tile was clearly
    fastest in the all-tiles timing on a B200 (bench.py --selector-study,
    K = 2560, operands from HBM; the runner-up at least 8% slower), the
    selector picks it."""
    names = [mr.gemm_f16_tile_name(t) for t in range(mr.gemm_f16_num_tiles())]
    for N in (512, 1152, 4096, 6144):
        for rt in (3, 10, 21, 32):
            picks = {mr.gemm_f16_select_tile(M, N, 2560) for M in (64 * (rt - 1) + 1, 64 * rt - 17, 64 * rt)}
            assert len(picks) == 1, (N, rt, picks)
    measured_best = {(1983, 1152): "256x128", (150, 1664): "64x64", (192, 1664): "64x64", (306, 1664): "64x64",
                     (700, 1664): "64x128", (1300, 1664): "128x128", (1983, 1664): "128x192",
                     (2048, 1664): "128x192", (448, 4096): "256x128", (700, 4096): "128x192",
                     (1983, 4096): "256x256", (2048, 4096): "256x256", (306, 6144): "128x128",
                     (448, 6144): "128x192", (1300, 6144): "256x256", (1983, 6144): "256x256",
                     (2048, 6144): "256x256"}
    for (M, N), name in measured_best.items():
        assert names[mr.gemm_f16_select_tile(M, N, 2560)] == name, (M, N)


def fused(A=A16, W=A16, logits=None, m=4, n=512, k=64, topk=10, idx=A16, ldo=10, ws=P(512), wsb=1 << 20):
    return mr.lib.router_gemv_topk(A, 64, W, 64, logits, 512, m, n, k, topk, idx, None, ldo, ws, wsb, 0, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ws=None), mr.MR_ERR_INVALID_ARG), (dict(idx=None), mr.MR_ERR_INVALID_ARG),
    (dict(topk=0), mr.MR_ERR_INVALID_ARG), (dict(topk=11), mr.MR_ERR_INVALID_ARG),
    (dict(topk=33, ldo=33), mr.MR_ERR_UNSUPPORTED), (dict(ws=P(272)), mr.MR_ERR_MISALIGNED),
    (dict(wsb=255), mr.MR_ERR_INVALID_ARG), (dict(wsb=256), mr.MR_ERR_INVALID_ARG),
    (dict(m=17), mr.MR_ERR_UNSUPPORTED), (dict(A=None), mr.MR_ERR_INVALID_ARG),
])
def test_fused_router_validation(kw, code):
    assert fused(**kw) == code


def test_fused_router_workspace_bytes():
    # head block, m x n tagged words, then (no logits passed) m x n fp32; each rounded up to 256 bytes
    assert mr.router_gemv_topk_workspace_bytes(4, 512, True) == 256 + 4 * 512 * 8
    assert mr.router_gemv_topk_workspace_bytes(4, 512, False) == 256 + 4 * 512 * 12
    assert mr.router_gemv_topk_workspace_bytes(1, 3, True) == 256 + 256
    assert mr.router_gemv_topk_workspace_bytes(1, 3, False) == 256 + 256 + 256
    assert mr.router_gemv_topk_workspace_bytes(0, 512, False) == 0
    need = mr.router_gemv_topk_workspace_bytes(4, 512, True)
    assert fused(logits=P(1024), wsb=need) == mr.MR_ERR_CUDA  # valid; no device here
    assert fused(logits=P(1024), wsb=need - 1) == mr.MR_ERR_INVALID_ARG


def test_grouped_validation():
    W = (P * 2)(256, 256)
    C = (P * 2)(256, 256)
    g = mr.lib.gemm_f16_grouped
    assert g(A16, 64, W, 64, C, 32, 4, 32, 64, 0, 0, 0, -1, None) == mr.MR_ERR_INVALID_ARG
    W65 = (P * 65)(*([256] * 65))
    C65 = (P * 65)(*([256] * 65))
    assert g(A16, 64, W65, 64, C65, 32, 4, 32, 64, 65, 0, 0, -1, None) == mr.MR_ERR_UNSUPPORTED
    Wn = (P * 2)(256, None)
    assert g(A16, 64, Wn, 64, C, 32, 4, 32, 64, 2, 0, 0, -1, None) == mr.MR_ERR_INVALID_ARG
    Wb = (P * 2)(256, 258)
    assert g(A16, 64, Wb, 64, C, 32, 4, 32, 64, 2, 0, 0, -1, None) == mr.MR_ERR_MISALIGNED
    assert g(A16, 64, W, 64, C, 32, 4, 32, 64, 2, 0, 0, -1, None) == mr.MR_ERR_CUDA  # valid; no device
    assert 0 <= mr.gemm_f16_grouped_select_tile(2048, 96, 2560, 36) < mr.gemm_f16_num_tiles()
    # A pair tile holds one group: several groups narrower than it go to the
    # packed one-CTA tiles (measured: 36 x N = 96 at M = 512, 12.4 us on
    # 128 x 96 against 13.1 us on the 256 x 128 pair).
    names = [mr.gemm_f16_tile_name(t) for t in range(mr.gemm_f16_num_tiles())]
    for M in (150, 512, 1024, 2048):
        assert not names[mr.gemm_f16_grouped_select_tile(M, 96, 2560, 36)].startswith("256x"), M
    assert names[mr.gemm_f16_grouped_select_tile(512, 96, 2560, 36)] == "128x96"


def test_cast_validation():
    c = mr.lib.cast_f32_bf16
    assert c(None, 8, A16, 8, 1, 8, None) == mr.MR_ERR_INVALID_ARG
    assert c(A16, 8, None, 8, 1, 8, None) == mr.MR_ERR_INVALID_ARG
    assert c(A16, 8, A16, 8, 0, 8, None) == mr.MR_ERR_INVALID_ARG
    assert c(A16, 4, A16, 8, 1, 8, None) == mr.MR_ERR_INVALID_ARG
    assert c(P(258), 8, A16, 8, 1, 8, None) == mr.MR_ERR_MISALIGNED
    assert c(A16, 8, P(257), 8, 1, 8, None) == mr.MR_ERR_MISALIGNED
    assert c(A16, 8, A16, 8, 1, 8, None) == mr.MR_ERR_CUDA  # valid; no device


def test_gate_flag_validation():
    assert gemv(flags=mr.MR_GEMV_SIGMOID) == mr.MR_ERR_CUDA          # accepted; no device
    assert gemv(flags=mr.MR_GEMV_SIGMOID | mr.MR_GEMV_PDL) == mr.MR_ERR_CUDA
    assert gemv(flags=4) == mr.MR_ERR_INVALID_ARG
    st = mr.lib.router_gemv_topk(A16, 64, A16, 64, None, 512, 4, 512, 64, 10, A16, None, 10, P(512),
                                 1 << 20, mr.MR_GEMV_SIGMOID, None)
    assert st == mr.MR_ERR_INVALID_ARG


def test_gemm_raster_validation():
    g = mr.lib.gemm_f16_ex
    assert g(A16, 64, A16, 64, A16, 32, 4, 32, 64, 0, 0, -1, -1, None) == mr.MR_ERR_INVALID_ARG
    assert g(A16, 64, A16, 64, A16, 32, 4, 32, 64, 0, 0, -1, 65, None) == mr.MR_ERR_INVALID_ARG
    assert g(A16, 64, A16, 64, A16, 32, 4, 32, 64, 0, 0, -1, 8, None) == mr.MR_ERR_CUDA  # valid; no device


def test_header_compiles_as_c99_and_links_from_c(tmp_path):
    """The boundary is a C ABI: the header compiles as strict C99 and a C
    program links against the library and gets the documented status codes
    from host-side validation (no device needed)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include "mrgemm.h"
int main(void) {
    int32_t out[8];
    int32_t idx[10];
    printf("%s\n", mr_version());
    printf("%d\n", (int)mrgemv_bf16(NULL, 64, NULL, 64, NULL, 32, 4, 32, 64, NULL));
    printf("%d\n", (int)mrgemv_bf16_plan(17, 512, 2560, 0, 148, 232448, out));
    printf("%d\n", (int)router_topk(NULL, 512, 1, 512, 10, idx, NULL, 10, NULL));
    printf("%d\n", (int)gemm_f16_select_tile(2048, 6144, 2560));
    printf("%s\n", mr_status_str(MR_ERR_MISALIGNED));
    return 0;
}
''')
    libdir = os.path.dirname(mr.LIB)
    exe = tmp_path / "abi"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.dirname(HEADER), str(src),
                    "-L", libdir, "-lmrgemm", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    lines = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    assert "sm_100a" in lines[0]
    assert int(lines[1]) == mr.MR_ERR_INVALID_ARG
    assert int(lines[2]) == mr.MR_ERR_UNSUPPORTED
    assert int(lines[3]) == mr.MR_ERR_INVALID_ARG
    assert mr.gemm_f16_tile_name(int(lines[4])) == "256x256"
    assert lines[5] == "MR_ERR_MISALIGNED"
