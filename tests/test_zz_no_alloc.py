"""router_gemv_topk_noalloc: the fused router for callers that cannot allocate
device memory (and so cannot pass a workspace).  Called through the C ABI and
checked against router_gemv_topk with a caller-owned workspace, on two calls
in a row: same indices, same values and the same logits, bit for bit (the two
entry points run the same kernel; only where the scratch lives differs)."""
import ctypes

import numpy as np
import pytest

import synth
from gpu_util import dev_bits, host, need_gpu, torch

import verify_weight_streaming_b200 as mr

pytestmark = pytest.mark.gpu


def _reference(A, W, m, n, k, topk):
    nbytes = mr.router_gemv_topk_workspace_bytes(m, n, True)
    ws = torch.zeros((nbytes + 3) // 4, dtype=torch.int32, device="cuda")
    logits = torch.empty((m, n), dtype=torch.float32, device="cuda")
    idx = torch.empty((m, topk), dtype=torch.int32, device="cuda")
    val = torch.empty((m, topk), dtype=torch.float32, device="cuda")
    mr.router_gemv_topk(A, W, topk, idx, val, logits=logits, workspace=ws)
    return host(logits), host(idx), host(val)


def _noalloc(A, W, m, n, k, topk, with_logits):
    logits = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda") if with_logits else None
    idx = torch.full((m, topk), -1, dtype=torch.int32, device="cuda")
    val = torch.full((m, topk), float("nan"), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = mr.lib.router_gemv_topk_noalloc(
        A.data_ptr(), A.stride(0), W.data_ptr(), W.stride(0),
        logits.data_ptr() if with_logits else None, n, m, n, k, topk,
        idx.data_ptr(), val.data_ptr(), topk, 0, stream)
    assert st == mr.MR_OK, mr.status_str(st)
    return (host(logits) if with_logits else None), host(idx), host(val)


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cases = [(16, 512, 2560, 10, 0), (3, 4864, 896, 32, 1)]
    for call, (m, n, k, topk, seed) in enumerate(cases):
        a = synth.normal_bits(3000 + seed, (m, k), "bf16", 1.0)
        w = synth.normal_bits(3100 + seed, (n, k), "bf16", 1.0 / np.sqrt(k))
        A, W = dev_bits(a), dev_bits(w)
        ref_l, ref_i, ref_v = _reference(A, W, m, n, k, topk)
        for with_logits in (False, True):
            l, i, v = _noalloc(A, W, m, n, k, topk, with_logits)
            assert np.array_equal(i, ref_i), (call, with_logits)
            assert np.array_equal(v.view(np.uint32), ref_v.view(np.uint32)), (call, with_logits)
            if with_logits:
                assert np.array_equal(l.view(np.uint32), ref_l.view(np.uint32))
    assert mr.mr_poll_errors() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cap = mr.lib.router_gemv_topk_noalloc_max_logits()
    # 12 bytes a logit (tagged word + fp32) after the 256-byte head block
    assert cap == (256 * 1024 - 256) // 12 // 64 * 64 == 21824
    assert mr.router_gemv_topk_workspace_bytes(16, cap // 16, False) <= 256 * 1024
    n = cap // 16 + 8  # 16 rows of n logits no longer fit
    A = torch.zeros((16, 64), dtype=torch.int16, device="cuda")
    W = torch.zeros((n, 64), dtype=torch.int16, device="cuda")
    idx = torch.empty((16, 10), dtype=torch.int32, device="cuda")
    st = mr.lib.router_gemv_topk_noalloc(A.data_ptr(), 64, W.data_ptr(), 64, None, n, 16, n, 64, 10,
                                         idx.data_ptr(), None, 10, 0, None)
    assert st == mr.MR_ERR_UNSUPPORTED


def _graph_nodes(graph) -> int:
    """Nodes of a captured (kept) torch CUDA graph, counted by the driver."""
    n = ctypes.c_size_t(0)
    cuda = ctypes.CDLL("libcuda.so.1")
    cuda.cuGraphGetNodes.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_size_t)]
    assert cuda.cuGraphGetNodes(ctypes.c_void_p(graph.raw_cuda_graph()), None, ctypes.byref(n)) == 0
    return n.value


def test_noalloc_invalid_call_puts_nothing_on_the_stream():
    """Every argument is checked before the tag array is cleared: an invalid call
    returns its error and adds no node to a stream being captured."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    m, n, k = 4, 512, 2560
    A = dev_bits(synth.normal_bits(3200, (m, k), "bf16", 1.0))
    W = dev_bits(synth.normal_bits(3201, (n, k), "bf16", 0.02))
    idx = torch.empty((m, 40), dtype=torch.int32, device="cuda")
    val = torch.empty((m, 40), dtype=torch.float32, device="cuda")
    x = torch.zeros(4, device="cuda")

    def call(topk=10, idx_ptr=None, kk=k, stream=None):
        return mr.lib.router_gemv_topk_noalloc(
            A.data_ptr(), k, W.data_ptr(), k, None, n, m, n, kk, topk,
            idx.data_ptr() if idx_ptr is None else idx_ptr, val.data_ptr(), 40, 0, stream)

    # A valid call outside capture: the first call on a device looks up the array.
    assert call() == mr.MR_OK
    torch.cuda.synchronize()
    bad = [(dict(topk=0), mr.MR_ERR_INVALID_ARG), (dict(topk=33), mr.MR_ERR_UNSUPPORTED),
           (dict(idx_ptr=idx.data_ptr() + 2), mr.MR_ERR_MISALIGNED), (dict(kk=12), mr.MR_ERR_MISALIGNED)]

    def capture(body):
        g = torch.cuda.CUDAGraph(keep_graph=True)
        s = torch.cuda.Stream()
        with torch.cuda.graph(g, stream=s):
            body(ctypes.c_void_p(s.cuda_stream))
            x.add_(1.0)
        return _graph_nodes(g)

    base = capture(lambda s: None)
    statuses = []
    bad_nodes = capture(lambda s: statuses.extend(call(stream=s, **kw) for kw, _ in bad))
    assert statuses == [want for _, want in bad]
    assert bad_nodes == base
    # A valid call inside the same kind of capture adds its nodes (memset + kernel).
    assert capture(lambda s: call(stream=s)) == base + 2
    assert mr.mr_poll_errors() == 0
