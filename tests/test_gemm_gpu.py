"""gemm_f16 (tcgen05) on the GPU: exactness on integer inputs, parity with the
fp64 oracle on the prompt-chunk shapes, and bitwise identity across tiles, M
and row order.

Pass bar: |C - C64| <= 1e-5 * sum|a*w| plus half an output ulp for f16/bf16
outputs.  At full sizes the oracle checks sampled rows and columns (computed
on the sliced operands, which gives the same per-element definition).
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import dev_bits, host, need_gpu, torch

import verify_weight_streaming_b200 as mr

pytestmark = pytest.mark.gpu

TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}
NP_OUT = {"f16": np.float16, "f32": np.float32}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()
    yield
    assert mr.mr_poll_errors() == 0


def run_gemm(a_bits, w_bits, in_fmt="f16", out_fmt="f16", tile=-1, ldc=None, lda=None):
    M, K = a_bits.shape
    N = w_bits.shape[0]
    A = dev_bits(a_bits, TORCH_DT[in_fmt])
    if lda is not None:
        buf = torch.zeros((M, lda), dtype=TORCH_DT[in_fmt], device="cuda")
        buf[:, :K] = A
        A = buf[:, :K]
    W = dev_bits(w_bits, TORCH_DT[in_fmt])
    ldc = ldc or (N + 7) // 8 * 8
    cbuf = torch.full((M + 1, ldc), float("nan"), dtype=TORCH_DT[out_fmt], device="cuda")
    C = cbuf[:M, :N]
    mr.gemm_f16(A, W, C, tile_id=tile)
    out = host(cbuf.float())
    assert np.isnan(out[M]).all() and np.isnan(out[:M, N:]).all(), "write outside C"
    raw = host(cbuf.view(torch.int16) if out_fmt != "f32" else cbuf.view(torch.int32))
    return out[:M, :N], raw[:M, :N]


def check(c, a_bits, w_bits, in_fmt, out_fmt, rows=None, cols=None):
    a = a_bits if rows is None else a_bits[rows]
    w = w_bits if cols is None else w_bits[cols]
    cc = c if rows is None else c[rows]
    cc = cc if cols is None else cc[:, cols]
    c64, s64 = oracle.matmul(a, in_fmt, w, in_fmt)
    ok, worst, where = oracle.check_matmul(cc, c64, s64, out_fmt)
    assert ok, f"worst |err|/tol = {worst:.3g} at {where}"


def test_single_tile_integer_exact():
    """One 128x32 tile, one K block: small integers make every step exact."""
    a = synth.integer_bits(1, (128, 64), "f16", -3, 3)
    w = synth.integer_bits(2, (32, 64), "f16", -3, 3)
    c, _ = run_gemm(a, w, out_fmt="f32", tile=0)
    ai = synth.bits_to_float32(a, "f16").astype(np.int64)
    wi = synth.bits_to_float32(w, "f16").astype(np.int64)
    assert np.array_equal(c.astype(np.int64), ai @ wi.T)


@pytest.mark.parametrize("tile", range(mr.gemm_f16_num_tiles()))
def test_every_tile_integer_exact_multi_block(tile):
    """Several M/N tiles and K blocks, ragged edges; all tiles exact on integers."""
    a = synth.integer_bits(3, (300, 200), "bf16", -7, 7)
    w = synth.integer_bits(4, (333, 200), "bf16", -7, 7)
    c, _ = run_gemm(a, w, in_fmt="bf16", out_fmt="f32", tile=tile)
    ai = synth.bits_to_float32(a, "bf16").astype(np.int64)
    wi = synth.bits_to_float32(w, "bf16").astype(np.int64)
    assert np.array_equal(c.astype(np.int64), ai @ wi.T)


@pytest.mark.parametrize("M", [512, 640, 768, 1024, 1983, 2048])
def test_narrow_n96_parity(M):
    """A[M,2560] x W[2560,96] f16 -> f16 (the Walbe projection shape)."""
    a, w = synth.narrow(M)
    c, _ = run_gemm(a, w)
    check(c, a, w, "f16", "f16")


@pytest.mark.parametrize("M,N", [(150, 512), (192, 640), (306, 1152), (448, 1664), (700, 4096),
                                 (1300, 6144), (1983, 6144), (2048, 4096)])
def test_chunk_shapes_sampled_parity(M, N):
    a, w = synth.chunk(M, N)
    c, _ = run_gemm(a, w)
    rng = np.random.default_rng(M + N)
    rows = np.unique(np.concatenate([rng.choice(M, 24, replace=False), [0, M - 1]]))
    cols = np.unique(np.concatenate([rng.choice(N, 48, replace=False), [0, N - 1]]))
    check(c, a, w, "f16", "f16", rows, cols)


def test_chunk_small_full_parity_all_dtypes():
    a, w = synth.chunk(150, 512)
    for in_fmt in ("f16", "bf16"):
        if in_fmt == "bf16":
            a = synth.normal_bits(71, (150, 2560), "bf16", 1.0)
            w = synth.normal_bits(72, (512, 2560), "bf16", 1.0 / np.sqrt(2560))
        for out_fmt in ("f16", "bf16", "f32"):
            c, _ = run_gemm(a, w, in_fmt=in_fmt, out_fmt=out_fmt)
            check(c, a, w, in_fmt, out_fmt)


@pytest.mark.parametrize("M,N,K", [(1, 1, 8), (5, 17, 72), (129, 100, 136), (64, 96, 2560),
                                   (200, 31, 1000), (257, 264, 64)])
def test_edges(M, N, K):
    a = synth.normal_bits(11 + M, (M, K), "f16", 1.0)
    w = synth.normal_bits(12 + N, (N, K), "f16", 1.0 / np.sqrt(K))
    for tile in (-1, 0, 5, 6, 7, 8):
        c, _ = run_gemm(a, w, tile=tile)
        check(c, a, w, "f16", "f16")


def test_strides_and_canaries():
    a, w = synth.chunk(300, 512)
    c, _ = run_gemm(a, w, ldc=528, lda=2568)
    check(c, a, w, "f16", "f16")


@pytest.mark.parametrize("M,N,fmt", [(1983, 96, "f16"), (306, 1152, "f16"), (700, 640, "bf16")])
def test_bitwise_identical_across_tiles_M_and_row_order(M, N, fmt):
    a = synth.normal_bits(21, (M, 2560), fmt, 1.0)
    w = synth.normal_bits(22, (N, 2560), fmt, 1.0 / np.sqrt(2560))
    _, ref = run_gemm(a, w, in_fmt=fmt, out_fmt=fmt, tile=0)
    for tile in range(1, mr.gemm_f16_num_tiles()):
        _, raw = run_gemm(a, w, in_fmt=fmt, out_fmt=fmt, tile=tile)
        assert np.array_equal(raw, ref), f"tile {mr.gemm_f16_tile_name(tile)} differs"
    _, auto = run_gemm(a, w, in_fmt=fmt, out_fmt=fmt)
    assert np.array_equal(auto, ref)
    for m in (1, 64, 127, 129, M // 2):
        for tile in (3, 6, 8):   # a 128-row, a 64-row and the two-CTA 256-row tile
            _, part = run_gemm(a[:m], w, in_fmt=fmt, out_fmt=fmt, tile=tile)
            assert np.array_equal(part, ref[:m]), f"prefix M={m} differs (tile {tile})"
    perm = np.random.default_rng(5).permutation(M)
    _, pr = run_gemm(a[perm], w, in_fmt=fmt, out_fmt=fmt, tile=5)
    assert np.array_equal(pr, ref[perm])


def test_f32_out_bitwise_across_tiles():
    a = synth.normal_bits(31, (260, 2560), "bf16", 1.0)
    w = synth.normal_bits(32, (6144, 2560), "bf16", 1.0 / np.sqrt(2560))[:700]
    _, ref = run_gemm(a, w, in_fmt="bf16", out_fmt="f32", tile=0)
    for tile in range(1, mr.gemm_f16_num_tiles()):
        _, raw = run_gemm(a, w, in_fmt="bf16", out_fmt="f32", tile=tile)
        assert np.array_equal(raw, ref)


def test_selector_choices_are_valid():
    for M in (150, 192, 306, 448, 512, 640, 700, 1024, 1300, 1983, 2048):
        for N in (96, 512, 640, 1152, 1664, 4096, 6144):
            t = mr.gemm_f16_select_tile(M, N, 2560)
            assert 0 <= t < mr.gemm_f16_num_tiles()


def run_grouped(a_bits, w_list, fmt="f16", out_fmt="f16", tile=-1):
    M, K = a_bits.shape
    N = w_list[0].shape[0]
    A = dev_bits(a_bits, TORCH_DT[fmt])
    Ws = [dev_bits(w, TORCH_DT[fmt]) for w in w_list]
    ldc = (N + 7) // 8 * 8
    bufs = [torch.full((M + 1, ldc), float("nan"), dtype=TORCH_DT[out_fmt], device="cuda") for _ in w_list]
    mr.gemm_f16_grouped(A, Ws, [b[:M, :N] for b in bufs], tile_id=tile)
    out = []
    for b in bufs:
        f = host(b.float())
        assert np.isnan(f[M]).all() and np.isnan(f[:M, N:]).all(), "write outside C"
        out.append(host(b.view(torch.int16) if out_fmt != "f32" else b.view(torch.int32))[:M, :N])
    return out


@pytest.mark.parametrize("M", [512, 1983])
def test_grouped_36_narrow_matches_single_calls(M):
    """The audit's chunk: one A, 36 W[96, 2560]; every output equals its single call."""
    a = synth.narrow(M)[0]
    ws = [synth.narrow(1, w_index=i)[1] for i in range(36)]
    grouped = run_grouped(a, ws)
    for i in (0, 1, 17, 35):
        _, ref = run_gemm(a, ws[i])
        assert np.array_equal(grouped[i], ref), f"group {i}"
    c = synth.bits_to_float32(grouped[7].view(np.uint16), "f16")
    check(c, a, ws[7], "f16", "f16")


@pytest.mark.parametrize("G,N,K", [(5, 48, 200), (3, 40, 136), (2, 300, 72), (1, 96, 2560), (64, 16, 64)])
def test_grouped_every_tile_bitwise(G, N, K):
    a = synth.normal_bits(61 + G, (257, K), "bf16", 1.0)
    ws = [synth.normal_bits(62 + 7 * g + N, (N, K), "bf16", 1.0 / np.sqrt(K)) for g in range(G)]
    refs = [run_gemm(a, w, in_fmt="bf16", out_fmt="bf16", tile=0)[1] for w in ws]
    for tile in range(-1, mr.gemm_f16_num_tiles()):
        outs = run_grouped(a, ws, fmt="bf16", out_fmt="bf16", tile=tile)
        for g in range(G):
            assert np.array_equal(outs[g], refs[g]), (tile, g)


@pytest.mark.parametrize("M,N,tile", [(700, 640, 0), (1983, 1152, 3), (300, 2000, 5), (129, 96, 2)])
def test_raster_orders_give_identical_bits(M, N, tile):
    """Tile order (the SLC-swizzle analogue) changes only the schedule."""
    a = synth.normal_bits(41, (M, 2560), "f16", 1.0)
    w = synth.normal_bits(42, (N, 2560), "f16", 1.0 / np.sqrt(2560))
    A, W = dev_bits(a, torch.float16), dev_bits(w, torch.float16)
    ldc = (N + 7) // 8 * 8
    ref = None
    for raster in (0, 1, 2, 3, 8, 64):
        C = torch.full((M, ldc), float("nan"), dtype=torch.float16, device="cuda")
        mr.gemm_f16(A, W, C[:, :N], tile_id=tile, raster=raster)
        raw = host(C.view(torch.int16))[:, :N]
        if ref is None:
            ref = raw
            check(synth.bits_to_float32(raw.view(np.uint16), "f16")[:64], a[:64], w, "f16", "f16")
        assert np.array_equal(raw, ref), raster


# ------------------------------------------------------ full-size parity
# Every element of the output against the fp64 oracle, at the full prompt-chunk
# sizes (the oracle takes tens of seconds on the host's cores for each).

def test_full_parity_1983x1152_f16():
    """The Wk chunk shape (M % 128 = 63, a tail tile), f16 in and out, auto tile."""
    a, w = synth.chunk(1983, 1152)
    c, _ = run_gemm(a, w)
    check(c, a, w, "f16", "f16")


def test_full_parity_1024x6144_bf16_to_f32():
    """The m-sweep's GEMM path: bf16 in, fp32 out, K = 2560, N = 6144."""
    a = synth.normal_bits(synth.seed_for(synth.WL_SWEEP, 0), (1024, 2560), "bf16", 1.0)
    w = synth.normal_bits(synth.seed_for(synth.WL_SWEEP, 1), (6144, 2560), "bf16", 1.0 / np.sqrt(2560))
    c, _ = run_gemm(a, w, in_fmt="bf16", out_fmt="f32")
    check(c, a, w, "bf16", "f32")


def test_full_parity_grouped_36_narrow_at_2048():
    """All 36 N = 96 outputs of one grouped launch at M = 2048, every element
    (the oracle runs once on the 36 weights stacked: the same per-element sum)."""
    a = synth.narrow(2048)[0]
    ws = [synth.narrow(1, w_index=i)[1] for i in range(36)]
    outs = run_grouped(a, ws)
    c = np.concatenate([synth.bits_to_float32(o.view(np.uint16), "f16") for o in outs], axis=1)
    check(c, a, np.concatenate(ws, axis=0), "f16", "f16")
