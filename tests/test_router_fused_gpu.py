"""router_gemv_topk (GEMV + top-k in one launch) against the two-launch path:
logits, indices and values bitwise equal; the workspace's tag array is all
zero again after every call."""
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


def workspace(m, n, with_logits):
    nbytes = mr.router_gemv_topk_workspace_bytes(m, n, with_logits)
    return torch.zeros((nbytes + 3) // 4, dtype=torch.int32, device="cuda")


def tags_are_zero(ws, m, n) -> bool:
    """The m x n tagged words after the 256-byte head block."""
    return not host(ws)[64:64 + 2 * m * n].any()


def two_launch(A, W, m, n, topk):
    C = torch.empty((m, n), dtype=torch.float32, device="cuda")
    idx = torch.empty((m, topk), dtype=torch.int32, device="cuda")
    val = torch.empty((m, topk), dtype=torch.float32, device="cuda")
    mr.mrgemv_bf16(A, W, C)
    mr.router_topk(C, topk, idx, val)
    return host(C), host(idx), host(val)


@pytest.mark.parametrize("m", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("with_logits", [True, False])
def test_fused_matches_two_launches(m, with_logits):
    a, w = synth.router(m)
    A, W = dev_bits(a), dev_bits(w)
    c_ref, i_ref, v_ref = two_launch(A, W, m, 512, 10)
    ws = workspace(m, 512, with_logits)
    idx = torch.full((m, 10), -1, dtype=torch.int32, device="cuda")
    val = torch.full((m, 10), float("nan"), dtype=torch.float32, device="cuda")
    logits = torch.empty((m, 512), dtype=torch.float32, device="cuda") if with_logits else None
    mr.router_gemv_topk(A, W, 10, idx, val, logits=logits, workspace=ws)
    assert np.array_equal(host(idx), i_ref)
    assert np.array_equal(host(val).view(np.uint32), v_ref.view(np.uint32))
    if with_logits:
        assert np.array_equal(host(logits).view(np.uint32), c_ref.view(np.uint32))
    assert tags_are_zero(ws, m, 512), "the selecting warps zero the tagged words"
    ri, _ = oracle.topk(c_ref, 10)
    assert np.array_equal(host(idx), ri)


@pytest.mark.parametrize("m,n,k,topk", [(5, 37, 136, 7), (16, 4864, 896, 32), (2, 6144, 2560, 10),
                                        (9, 3, 8, 3), (16, 149, 1024, 1)])
def test_other_shapes(m, n, k, topk):
    a = synth.normal_bits(500 + n, (m, k), "bf16", 1.0)
    w = synth.normal_bits(600 + k, (n, k), "bf16", 1.0 / np.sqrt(k))
    A, W = dev_bits(a), dev_bits(w)
    c_ref, i_ref, v_ref = two_launch(A, W, m, n, topk)
    ws = workspace(m, n, False)
    idx = torch.empty((m, topk), dtype=torch.int32, device="cuda")
    val = torch.empty((m, topk), dtype=torch.float32, device="cuda")
    mr.router_gemv_topk(A, W, topk, idx, val, workspace=ws)
    assert np.array_equal(host(idx), i_ref)
    assert np.array_equal(host(val).view(np.uint32), v_ref.view(np.uint32))
    assert tags_are_zero(ws, m, n)
    c64, s64 = oracle.matmul(a, "bf16", w, "bf16")
    ok, worst, _ = oracle.check_matmul(c_ref, c64, s64)
    assert ok, worst


def test_many_calls_graph_and_pdl_reuse_one_workspace():
    ms = [16, 1, 8, 4, 2]
    ins = []
    for i, m in enumerate(ms):
        a = synth.normal_bits(900 + i, (m, 2560), "bf16", 1.0)
        w = synth.normal_bits(950 + i, (512, 2560), "bf16", 0.02)
        ins.append((m, dev_bits(a), dev_bits(w)))
    refs = [two_launch(A, W, m, 512, 10) for m, A, W in ins]
    ws = workspace(16, 512, False)
    outs = [(torch.empty((m, 10), dtype=torch.int32, device="cuda"),
             torch.empty((m, 10), dtype=torch.float32, device="cuda")) for m, _, _ in ins]
    s = torch.cuda.Stream()
    for _ in range(20):
        with torch.cuda.stream(s):
            for (m, A, W), (i, v) in zip(ins, outs):
                mr.router_gemv_topk(A, W, 10, i, v, workspace=ws, flags=mr.MR_GEMV_PDL)
    torch.cuda.synchronize()
    for (c, ir, vr), (i, v) in zip(refs, outs):
        assert np.array_equal(host(i), ir)
        assert np.array_equal(host(v).view(np.uint32), vr.view(np.uint32))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for (m, A, W), (i, v) in zip(ins, outs):
            mr.router_gemv_topk(A, W, 10, i, v, workspace=ws, flags=mr.MR_GEMV_PDL)
    for i, v in outs:
        i.fill_(-1)
    for _ in range(10):
        g.replay()
    torch.cuda.synchronize()
    for (c, ir, vr), (i, v) in zip(refs, outs):
        assert np.array_equal(host(i), ir)
    assert tags_are_zero(ws, 16, 512)


def test_fused_and_two_launch_calls_of_any_m_share_one_workspace():
    """The two-launch form keeps its logits at the end of the workspace, clear
    of the tag array of any call the workspace was sized for."""
    ws = workspace(16, 512, False)
    ws.fill_(0)
    seq = [(16, 0), (1, mr.MR_ROUTER_TWO_LAUNCH), (16, 0), (4, mr.MR_ROUTER_TWO_LAUNCH), (8, 0), (16, 0)]
    for i, (m, form) in enumerate(seq):
        a = synth.normal_bits(1300 + i, (m, 2560), "bf16", 1.0)
        w = synth.normal_bits(1350 + i, (512, 2560), "bf16", 0.02)
        A, W = dev_bits(a), dev_bits(w)
        _, ir, vr = two_launch(A, W, m, 512, 10)
        idx = torch.empty((m, 10), dtype=torch.int32, device="cuda")
        val = torch.empty((m, 10), dtype=torch.float32, device="cuda")
        mr.router_gemv_topk(A, W, 10, idx, val, workspace=ws, flags=mr.MR_GEMV_PDL | form)
        assert np.array_equal(host(idx), ir), (i, m, form)
        assert np.array_equal(host(val).view(np.uint32), vr.view(np.uint32)), (i, m, form)
        assert tags_are_zero(ws, 16, 512), (i, m, form)


@pytest.mark.parametrize("m", [1, 5, 16])
@pytest.mark.parametrize("with_logits", [True, False])
def test_two_launch_flag_matches_fused_and_separate_calls(m, with_logits):
    """MR_ROUTER_TWO_LAUNCH: one call, GEMV kernel then top-k kernel: the same bits."""
    a, w = synth.router(m)
    A, W = dev_bits(a), dev_bits(w)
    c_ref, i_ref, v_ref = two_launch(A, W, m, 512, 10)
    ws = workspace(m, 512, with_logits)
    ws.fill_(-1)   # neither the head block nor the tag array is used by this form
    idx = torch.full((m, 10), -1, dtype=torch.int32, device="cuda")
    val = torch.full((m, 10), float("nan"), dtype=torch.float32, device="cuda")
    logits = torch.empty((m, 512), dtype=torch.float32, device="cuda") if with_logits else None
    mr.router_gemv_topk(A, W, 10, idx, val, logits=logits, workspace=ws,
                        flags=mr.MR_GEMV_PDL | mr.MR_ROUTER_TWO_LAUNCH)
    assert np.array_equal(host(idx), i_ref)
    assert np.array_equal(host(val).view(np.uint32), v_ref.view(np.uint32))
    if with_logits:
        assert np.array_equal(host(logits).view(np.uint32), c_ref.view(np.uint32))
    else:
        off = (ws.numel() * 4 - m * 512 * 4) // 256 * 256 // 4   # the last m * n * 4 bytes
        got = host(ws)[off:off + m * 512].view(np.float32).reshape(m, 512)
        assert np.array_equal(got.view(np.uint32), c_ref.view(np.uint32))
    with pytest.raises(mr.MrError):
        mr.router_gemv_topk(A, W, 10, idx, val, workspace=ws, flags=mr.MR_GEMV_SIGMOID)


@pytest.mark.parametrize("heavy", [False, True])
def test_fused_ties_inf_nan_through_the_tags(heavy):
    """Special logits cross the tag array bit for bit: ties (equal W rows),
    +-inf (an inf weight times a nonzero a) and NaN (inf times a zero a).
    With `heavy`, 40 equal rows at the top leave more than 32 candidates, so
    the selection takes its tie fallback inside the fused kernel."""
    m, n, k = 4, 512, 64
    a = synth.normal_bits(1400, (m, k), "bf16", 1.0)
    w = synth.normal_bits(1401, (n, k), "bf16", 0.05)
    top = range(100, 140) if heavy else (10, 300, 301)
    w[5] = synth.normal_bits(1402, (1, k), "bf16", 1.0)[0]
    for j in top:
        w[j] = w[5]                      # equal logits: ties go to the lower index
    w[7] = 0
    w[7, 0] = 0x7F80                     # +inf weight
    w[8] = 0
    w[8, 1] = 0xFF80                     # -inf weight
    a[2, 0] = 0                          # row 2: inf * 0 = NaN at column 7
    A, W = dev_bits(a), dev_bits(w)
    c_ref, i_ref, v_ref = two_launch(A, W, m, n, 10)
    assert np.isnan(c_ref[2, 7]) and np.isinf(c_ref[0, 7]) and np.isinf(c_ref[0, 8])
    ws = workspace(m, n, False)
    idx = torch.full((m, 10), -1, dtype=torch.int32, device="cuda")
    val = torch.full((m, 10), float("nan"), dtype=torch.float32, device="cuda")
    mr.router_gemv_topk(A, W, 10, idx, val, workspace=ws, flags=mr.MR_GEMV_PDL)
    assert np.array_equal(host(idx), i_ref)
    assert np.array_equal(host(val).view(np.uint32), v_ref.view(np.uint32))
    ri, rv = oracle.topk(c_ref, 10)
    assert np.array_equal(host(idx), ri)
    assert np.array_equal(host(val).view(np.uint32), rv.view(np.uint32))
    assert tags_are_zero(ws, m, n)
