"""mrgemv_bf16 on the GPU against the fp64 oracle, plus bitwise batch invariance.

Pass bar (per element): |C_gpu - C64| <= 1e-5 * sum|a*w|.  Bitwise: row i of
the output is the same for every m in 1..16 and every position in A, with and
without programmatic dependent launch.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import dev_bits, host, need_gpu, padded, torch

import verify_weight_streaming_b200 as mr

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()
    yield
    assert mr.mr_poll_errors() == 0


def run_gemv(a_bits, w_bits, flags=0, ldc=None, lda=None, ldw=None):
    m, k = a_bits.shape
    n = w_bits.shape[0]
    A = dev_bits(a_bits)
    if lda is not None:
        buf, A2 = padded(m, k, lda, torch.int16, 0x7FC0)
        A2.copy_(A)
        A = A2
    W = dev_bits(w_bits)
    if ldw is not None:
        buf, W2 = padded(n, k, ldw, torch.int16, 0x7FC0)
        W2.copy_(W)
        W = W2
    ldc = ldc or n
    cbuf = torch.full((m + 1, ldc), float("nan"), dtype=torch.float32, device="cuda")
    C = cbuf[:m, :n]
    mr.mrgemv_bf16(A, W, C, flags=flags)
    out = host(cbuf)
    # canaries: padding columns and the spare row are untouched
    assert np.isnan(out[:m, n:]).all() and np.isnan(out[m]).all()
    return out[:m, :n]


def check(c, a_bits, w_bits):
    c64, s64 = oracle.matmul(a_bits, "bf16", w_bits, "bf16")
    ok, worst, where = oracle.check_matmul(c, c64, s64)
    assert ok, f"worst |err|/tol = {worst:.3g} at {where}"
    return worst


@pytest.mark.parametrize("m", [1, 2, 4, 8, 16])
def test_ffn_shape_parity(m):
    """A[m,896] x W[896,4864] (the KAT's Qwen FFN inner dim)."""
    a, w = synth.gemv_ffn(m)
    check(run_gemv(a, w), a, w)


@pytest.mark.parametrize("m", [1, 2, 4, 8, 16])
def test_router_shape_parity(m):
    """A[m,2560] x W_r[2560,512] (the 2.6 MB router)."""
    a, w = synth.router(m)
    check(run_gemv(a, w), a, w)


def test_sweep_shape_parity_ring_refill():
    """K=2560, N=6144: more column groups than ring slots, so slots are refilled."""
    a = synth.normal_bits(synth.seed_for(synth.WL_SWEEP, 0), (16, 2560), "bf16", 1.0)
    w = synth.normal_bits(synth.seed_for(synth.WL_SWEEP, 1), (6144, 2560), "bf16", 1.0 / np.sqrt(2560))
    check(run_gemv(a, w), a, w)


@pytest.mark.parametrize("m,n,k", [
    (1, 1, 8), (3, 5, 24), (5, 33, 136), (16, 147, 1024), (7, 149, 2048), (2, 300, 520),
    (16, 1000, 4096), (9, 2, 8), (11, 7, 4088),
])
def test_ragged_shapes(m, n, k):
    a = synth.normal_bits(100 + k, (m, k), "bf16", 1.0)
    w = synth.normal_bits(200 + n, (n, k), "bf16", 1.0 / np.sqrt(k))
    check(run_gemv(a, w), a, w)


def test_strided_operands_and_canaries():
    a, w = synth.gemv_ffn(6, k=896, n=1000)
    c = run_gemv(a, w, ldc=1016, lda=904, ldw=912)
    check(c, a, w)


def test_integer_inputs_are_exact():
    """Small integers: every partial sum is an integer below 2^24, so fp32 is exact."""
    for (m, n, k) in [(16, 300, 896), (4, 64, 2560)]:
        a = synth.integer_bits(5, (m, k), "bf16", -15, 15)
        w = synth.integer_bits(6, (n, k), "bf16", -15, 15)
        c = run_gemv(a, w)
        c64, _ = oracle.matmul(a, "bf16", w, "bf16")
        assert np.array_equal(c.astype(np.float64), c64)


@pytest.mark.parametrize("shape", ["ffn", "router", "ragged"])
def test_rows_bitwise_identical_across_m(shape):
    if shape == "ffn":
        a, w = synth.gemv_ffn(16)
    elif shape == "router":
        a, w = synth.router(16)
    else:
        a = synth.normal_bits(9, (16, 1032), "bf16", 1.0)
        w = synth.normal_bits(10, (77, 1032), "bf16", 0.03)
    full = run_gemv(a, w)
    for m in range(1, 16):
        part = run_gemv(a[:m], w)
        assert np.array_equal(part.view(np.uint32), full[:m].view(np.uint32)), f"m={m}"
    # a row placed anywhere in the window gives the same bits
    perm = np.random.default_rng(0).permutation(16)
    pc = run_gemv(a[perm], w)
    assert np.array_equal(pc.view(np.uint32), full[perm].view(np.uint32))
    for i in (0, 5, 15):
        single = run_gemv(a[i:i + 1], w)
        assert np.array_equal(single.view(np.uint32), full[i:i + 1].view(np.uint32))


# Row buckets of 1-2 rows advance two rows per packed fp32 FMA on converted
# operands; buckets of 4 and more use the mixed-precision FMA on the bf16
# operands.  The two are the same arithmetic, which these check on the values
# where hardware shortcuts would show: subnormals, infinities and NaN.
_SMALL_POW2 = np.array([0x0000, 0x3F80, 0xBF80, 0x4000, 0xC000, 0x4080, 0xC080], np.uint16)  # 0, +-1, +-2, +-4


def _subnormal_bits(rng, shape):
    """bf16 subnormals: exponent field 0, mantissa 1..127, either sign."""
    return ((rng.integers(0, 2, size=shape) << 15) | rng.integers(1, 128, size=shape)).astype(np.uint16)


@pytest.mark.parametrize("side", ["A", "W"])
def test_subnormal_operands_are_exact_at_every_m(side):
    """Subnormal bf16 times 0, +-1, +-2 or +-4: every product and partial sum is
    a multiple of 2^-133 with fewer than 2^24 of them, so the fp32 result is
    exact (no operand or result may be flushed to zero), at every m."""
    rng = np.random.default_rng(41 if side == "A" else 42)
    m_max, n, k = 16, 40, 264
    if side == "A":
        a = _subnormal_bits(rng, (m_max, k))
        w = _SMALL_POW2[rng.integers(0, len(_SMALL_POW2), size=(n, k))]
    else:
        a = _SMALL_POW2[rng.integers(0, len(_SMALL_POW2), size=(m_max, k))]
        w = _subnormal_bits(rng, (n, k))
    for m in (1, 2, 3, 4, 5, 8, 9, 16):
        c = run_gemv(a[:m], w)
        c64, _ = oracle.matmul(a[:m], "bf16", w, "bf16")
        assert np.count_nonzero(c64) > m * n // 2
        assert np.array_equal(c.astype(np.float64), c64), f"m={m}"


def test_inf_nan_rows_bitwise_identical_across_m():
    """Infinities and NaN in A and W: the same bits at every m (NaN included),
    and NaN / +-inf exactly where the oracle has them."""
    k, n = 520, 96
    a = synth.normal_bits(51, (16, k), "bf16", 1.0)
    w = synth.normal_bits(52, (n, k), "bf16", 1.0 / np.sqrt(k))
    a[1, 7] = 0x7F80    # +inf: row 1 is +-inf or NaN wherever W[:, 7] != 0
    a[4, 100] = 0xFF80  # -inf
    a[4, 300] = 0x7F80  # and +inf in the same row: NaN where both products are finite-signed
    a[6, 9] = 0x7FC0    # NaN
    a[11, 513] = 0xFFC1  # NaN with a payload and the sign set
    w[3, 200] = 0x7F80  # column 3: +inf in every row with a nonzero A[:, 200]
    w[50, 17] = 0x0000
    a[13, 17] = 0x7F80  # inf times zero in column 50: NaN
    full = run_gemv(a, w)
    c64, _ = oracle.matmul(a, "bf16", w, "bf16")
    assert np.array_equal(np.isnan(full), np.isnan(c64))
    assert np.array_equal(np.isposinf(full), np.isposinf(c64))
    assert np.array_equal(np.isneginf(full), np.isneginf(c64))
    assert np.isnan(full).any() and np.isinf(full).any()
    for m in range(1, 16):
        part = run_gemv(a[:m], w)
        assert np.array_equal(part.view(np.uint32), full[:m].view(np.uint32)), f"m={m}"
    for i in (1, 4, 6, 11, 13):
        single = run_gemv(a[i:i + 1], w)
        assert np.array_equal(single.view(np.uint32), full[i:i + 1].view(np.uint32)), f"row {i}"


def test_pdl_flag_gives_identical_bits():
    a, w = synth.router(8)
    plain = run_gemv(a, w)
    pdl = run_gemv(a, w, flags=mr.MR_GEMV_PDL)
    assert np.array_equal(plain.view(np.uint32), pdl.view(np.uint32))
    a, w = synth.gemv_ffn(16)
    assert np.array_equal(run_gemv(a, w).view(np.uint32),
                          run_gemv(a, w, flags=mr.MR_GEMV_PDL).view(np.uint32))


def test_bounded_wait_selftest_reports_and_context_survives():
    assert mr.mr_poll_errors() == 0
    mr.mr_selftest_wait_timeout(2000)
    flags = mr.mr_poll_errors()
    assert flags == mr.MR_DEVERR_SELFTEST
    assert mr.mr_poll_errors() == 0
    a, w = synth.router(2)
    check(run_gemv(a, w), a, w)


@pytest.mark.parametrize("m", [1, 8, 16])
def test_sweep_shape_pdl_budget(m):
    """K=2560, N=6144 under the PDL shared-memory budget: one ring slot, many refills."""
    a = synth.normal_bits(synth.seed_for(synth.WL_SWEEP, 0), (m, 2560), "bf16", 1.0)
    w = synth.normal_bits(synth.seed_for(synth.WL_SWEEP, 1), (6144, 2560), "bf16", 1.0 / np.sqrt(2560))
    c = run_gemv(a, w, flags=mr.MR_GEMV_PDL)
    check(c, a, w)
    assert np.array_equal(c.view(np.uint32), run_gemv(a, w).view(np.uint32))


def test_back_to_back_pdl_launches_in_a_graph():
    """Dependent launches overlap; every output must still match its own inputs."""
    shapes = [(16, 2560, 512), (8, 896, 4864), (1, 2560, 6144), (16, 2560, 6144), (4, 2560, 512)]
    ins, outs = [], []
    for i, (m, k, n) in enumerate(shapes):
        a = synth.normal_bits(700 + i, (m, k), "bf16", 1.0)
        w = synth.normal_bits(800 + i, (n, k), "bf16", 1.0 / np.sqrt(k))
        ins.append((a, w, dev_bits(a), dev_bits(w)))
        outs.append(torch.empty((m, n), dtype=torch.float32, device="cuda"))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for (a, w, A, W), C in zip(ins, outs):
            mr.mrgemv_bf16(A, W, C, flags=mr.MR_GEMV_PDL)
    torch.cuda.synchronize()
    eager = [host(C).copy() for C in outs]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for (a, w, A, W), C in zip(ins, outs):
            mr.mrgemv_bf16(A, W, C, flags=mr.MR_GEMV_PDL)
    for C in outs:
        C.fill_(float("nan"))
    g.replay()
    g.replay()
    for (a, w, _, _), C, e in zip(ins, outs, eager):
        c = host(C)
        check(c, a, w)
        assert np.array_equal(c.view(np.uint32), e.view(np.uint32))


def test_binding_launches_on_the_current_torch_stream():
    s = torch.cuda.Stream()
    assert mr._current_stream_handle() == torch.cuda.current_stream().cuda_stream
    with torch.cuda.stream(s):
        assert mr._current_stream_handle() == s.cuda_stream
    assert mr._current_stream_handle() == torch.cuda.current_stream().cuda_stream
