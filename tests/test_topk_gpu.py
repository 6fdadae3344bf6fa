"""router_topk on the GPU: indices bit-exact against the oracle's top-k of the
same fp32 logits, values bitwise equal to the logits at those indices."""
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


def gpu_topk(logits: np.ndarray, k: int, with_val=True, ldo=None, ldl=None):
    m, n = logits.shape
    ldl = ldl or n
    lbuf = torch.full((m, ldl), float("nan"), dtype=torch.float32, device="cuda")
    lbuf[:, :n] = torch.from_numpy(np.ascontiguousarray(logits)).cuda()
    L = lbuf[:, :n]
    ldo = ldo or k
    ibuf = torch.full((m + 1, ldo), -7, dtype=torch.int32, device="cuda")
    vbuf = torch.full((m + 1, ldo), 123.0, dtype=torch.float32, device="cuda")
    mr.router_topk(L, k, ibuf[:m, :k], vbuf[:m, :k] if with_val else None)
    ih, vh = host(ibuf), host(vbuf)
    assert (ih[m] == -7).all() and (ih[:m, k:] == -7).all()
    assert (vh[m] == 123.0).all() and (vh[:m, k:] == 123.0).all()
    if not with_val:
        assert (vh == 123.0).all()
    return ih[:m, :k], vh[:m, :k]


def check(logits, k, **kw):
    idx, val = gpu_topk(logits, k, **kw)
    ri, rv = oracle.topk(logits, k)
    assert np.array_equal(idx, ri)
    if kw.get("with_val", True):
        assert np.array_equal(val.view(np.uint32), logits[np.arange(len(logits))[:, None], idx].view(np.uint32))


@pytest.mark.parametrize("m", [1, 2, 4, 8, 16])
def test_router_window_on_gpu_logits(m):
    """The router step: GPU GEMV logits -> GPU top-10, checked on those same logits."""
    a, w = synth.router(m)
    A, W = dev_bits(a), dev_bits(w)
    C = torch.empty((m, 512), dtype=torch.float32, device="cuda")
    mr.mrgemv_bf16(A, W, C)
    logits = host(C)
    check(logits, 10)


@pytest.mark.parametrize("n,k", [(512, 10), (1, 1), (7, 7), (31, 10), (128, 32), (129, 1),
                                 (1000, 17), (2048, 32), (2049, 10), (5000, 10), (4097, 32)])
def test_shapes(n, k):
    x = synth.bits_to_float32(synth.normal_bits(400 + n, (6, n), "bf16", 1.0), "bf16")
    check(x, k)


def test_planted_ties_lower_index_wins():
    x = synth.choice_f32(41, (16, 512), [-1.0, 0.0, 1.0, 2.0])
    check(x, 10)
    x = synth.choice_f32(42, (9, 700), [3.0, 3.0, 3.0, -3.0])
    check(x, 32)
    # duplicated weight columns give bitwise-equal logits
    a, w = synth.router(4)
    w = w.copy()
    w[300] = w[7]
    w[450] = w[7]
    A, W = dev_bits(a), dev_bits(w)
    C = torch.empty((4, 512), dtype=torch.float32, device="cuda")
    mr.mrgemv_bf16(A, W, C)
    logits = host(C)
    assert (logits[:, 300] == logits[:, 7]).all()
    check(logits, 10)


def test_signed_zero_nan_inf():
    row = np.array([0.0, -0.0, 1.0, np.nan, -np.inf, np.inf, -0.0, np.nan, 1.0, -5.0] * 7,
                   dtype=np.float32)
    x = np.stack([row, -row, np.zeros_like(row), -np.zeros_like(row)])
    check(x, 32)
    check(x, 10)


def test_many_rows_strides_and_no_values():
    x = synth.bits_to_float32(synth.normal_bits(55, (300, 512), "bf16", 1.0), "bf16")
    check(x, 10, ldo=13, ldl=520)
    check(x, 10, with_val=False)
