"""The verify window's adjacent steps on the GPU: the bf16 cast of the
window's rows and the shared expert's scalar gate (n = 1 GEMV + sigmoid),
against the oracle; and the cast -> router GEMV -> top-10 chain end to end."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import dev_bits, host, need_gpu, torch

import verify_weight_streaming_b200 as mr

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()
    yield
    assert mr.mr_poll_errors() == 0


def special_rows(rows, cols, seed):
    """fp32 values with bf16 halfway cases, near-overflow, subnormals and signed zeros."""
    rng = np.random.default_rng(seed)
    base = rng.standard_normal((rows, cols)).astype(np.float32)
    bits = base.view(np.uint32)
    bits[:, ::7] = (bits[:, ::7] & 0xFFFF0000) | 0x8000          # exact halfway points
    bits[:, 1::11] = (bits[:, 1::11] & 0xFFFF0000) | 0x7FFF       # just below halfway
    bits[:, 2::13] = (bits[:, 2::13] & 0xFFFF0000) | 0x8001       # just above halfway
    out = bits.view(np.float32)
    out[:, 3::17] = np.float32(3.3e38)                              # rounds to inf or max
    out[:, 4::19] = np.float32(1e-40)                               # subnormal
    out[:, 5::23] = -0.0
    return out


def gpu_cast(x, ldy=None, ldx=None):
    rows, cols = x.shape
    ldx = ldx or cols
    xb = torch.full((rows, ldx), float("nan"), dtype=torch.float32, device="cuda")
    xb[:, :cols] = torch.from_numpy(x).cuda()
    ldy = ldy or cols
    yb = torch.full((rows + 1, ldy), 0x1234, dtype=torch.int16, device="cuda")
    mr.cast_f32_bf16(xb[:, :cols], yb[:rows, :cols])
    y = host(yb).view(np.uint16)
    assert (y[rows] == 0x1234).all() and (y[:rows, cols:] == 0x1234).all()
    return y[:rows, :cols]


@pytest.mark.parametrize("rows,cols,ldx,ldy", [(16, 2560, None, None), (5, 896, None, None),
                                               (3, 37, 40, 48), (7, 8, None, None), (1, 1, None, None),
                                               (2, 1000, 1004, 1000)])
def test_cast_matches_oracle(rows, cols, ldx, ldy):
    x = special_rows(rows, cols, rows * cols)
    y = gpu_cast(x, ldy=ldy, ldx=ldx)
    assert np.array_equal(y, oracle.cast_f32_bf16(x))


def test_cast_nan_stays_nan():
    x = np.array([[np.nan, -np.nan, np.inf, -np.inf, 1.0, 2.0, 3.0, 4.0]], dtype=np.float32)
    y = gpu_cast(x)
    assert ((y[0, :2] & 0x7F80) == 0x7F80).all() and (y[0, :2] & 0x7F).all()
    assert np.array_equal(y[0, 2:], oracle.cast_f32_bf16(x)[0, 2:])


@pytest.mark.parametrize("m", [1, 2, 3, 8, 16])
def test_shared_expert_gate(m):
    """n = 1 multi-row GEMV with the sigmoid in the same launch."""
    a = synth.normal_bits(811, (16, 2560), "bf16", 1.0)[:m]
    w = synth.normal_bits(812, (1, 2560), "bf16", 0.02)
    A, W = dev_bits(a), dev_bits(w)
    C = torch.full((m, 1), float("nan"), dtype=torch.float32, device="cuda")
    mr.mrgemv_bf16(A, W, C, flags=mr.MR_GEMV_SIGMOID)
    g = host(C).astype(np.float64)
    c64, s64 = oracle.matmul(a, "bf16", w, "bf16")
    err = np.abs(g - oracle.sigmoid(c64))
    assert (err <= oracle.gate_tolerance(c64, s64)).all(), err.max()
    # the gate's bits are those of the full-window call, row by row
    A16 = dev_bits(synth.normal_bits(811, (16, 2560), "bf16", 1.0))
    C16 = torch.empty((16, 1), dtype=torch.float32, device="cuda")
    mr.mrgemv_bf16(A16, W, C16, flags=mr.MR_GEMV_SIGMOID)
    assert np.array_equal(host(C16)[:m].view(np.uint32), host(C).view(np.uint32))


def test_gate_on_wide_output_and_pdl():
    a, w = synth.router(8)
    A, W = dev_bits(a), dev_bits(w)
    C = torch.empty((8, 512), dtype=torch.float32, device="cuda")
    mr.mrgemv_bf16(A, W, C, flags=mr.MR_GEMV_SIGMOID | mr.MR_GEMV_PDL)
    c64, s64 = oracle.matmul(a, "bf16", w, "bf16")
    assert (np.abs(host(C) - oracle.sigmoid(c64)) <= oracle.gate_tolerance(c64, s64)).all()


def test_window_chain_cast_gemv_topk():
    """fp32 hidden rows -> bf16 cast -> router GEMV -> top-10, against the oracle chain."""
    m = 16
    h = synth.bits_to_float32(synth.normal_bits(901, (m, 2560), "f16", 1.0), "f16") * np.float32(1.37)
    _, w = synth.router(m)
    H = torch.from_numpy(h).cuda()
    A = torch.empty((m, 2560), dtype=torch.int16, device="cuda")
    mr.cast_f32_bf16(H, A)
    a_bits = host(A).view(np.uint16)
    assert np.array_equal(a_bits, oracle.cast_f32_bf16(h))
    W = dev_bits(w)
    C = torch.empty((m, 512), dtype=torch.float32, device="cuda")
    idx = torch.empty((m, 10), dtype=torch.int32, device="cuda")
    mr.mrgemv_bf16(A, W, C)
    mr.router_topk(C, 10, idx)
    c = host(C)
    c64, s64 = oracle.matmul(a_bits, "bf16", w, "bf16")
    ok, worst, _ = oracle.check_matmul(c, c64, s64)
    assert ok, worst
    assert np.array_equal(host(idx), oracle.topk(c, 10)[0])
