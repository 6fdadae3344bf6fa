"""The column-split router's kernels on one GPU: G shards emulated in turn.

For each shard the GEMV runs on its block of weight rows (a pointer offset)
and router_topk_ex takes its top-k with global indices; router_topk_merge then
merges the G candidate lists.  The result must equal the one-device router
(mrgemv_bf16 on all columns, then router_topk) bit for bit, and the oracle's
top-k of the GPU's own logits.  Also: each shard's logits equal the matching
columns of the full call bit for bit (a logit depends only on its row of A,
its row of Wt and k).
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import dev_bits, host, need_gpu, torch

import verify_weight_streaming_b200 as mr
from verify_weight_streaming_b200 import sharded

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()
    yield
    assert mr.mr_poll_errors() == 0


def _split_router(A, W, n, topk, world):
    m = A.shape[0]
    cand_i = torch.full((world, m, topk), -1, dtype=torch.int32, device="cuda")
    cand_v = torch.zeros((world, m, topk), dtype=torch.float32, device="cuda")
    parts = []
    for r in range(world):
        b, e = sharded.shard_columns(n, world, r)
        lg = torch.empty((m, e - b), dtype=torch.float32, device="cuda")
        mr.mrgemv_bf16(A, W[b:e], lg, flags=mr.MR_GEMV_PDL)
        kl = sharded.local_topk(e - b, topk)
        mr.router_topk_ex(lg, kl, cand_i[r, :, :kl], cand_v[r, :, :kl], index_base=b)
        parts.append(lg)
    idx = torch.empty((m, topk), dtype=torch.int32, device="cuda")
    val = torch.empty((m, topk), dtype=torch.float32, device="cuda")
    mr.router_topk_merge(cand_v, cand_i, topk, idx, val)
    return host(idx), host(val), [host(p) for p in parts]


def _one_device(A, W, n, topk):
    m = A.shape[0]
    lg = torch.empty((m, n), dtype=torch.float32, device="cuda")
    mr.mrgemv_bf16(A, W, lg)
    idx = torch.empty((m, topk), dtype=torch.int32, device="cuda")
    val = torch.empty((m, topk), dtype=torch.float32, device="cuda")
    mr.router_topk(lg, topk, idx, val)
    return host(idx), host(val), host(lg)


@pytest.mark.parametrize("world", [2, 3, 4, 8])
@pytest.mark.parametrize("case", ["router", "ties"])
def test_split_router_equals_one_device(world, case):
    if case == "router":
        a, w = synth.router(16)
        topk = 10
    else:
        a = synth.choice_bits(51, (9, 256), "bf16", [-1, 0, 1])
        w = synth.choice_bits(52, (96, 256), "bf16", [-1, 0, 1])
        for r in range(1, world):          # duplicate columns across every boundary
            lo = sharded.shard_columns(96, world, r)[0]
            w[lo] = w[lo - 1]
        topk = 16
    n = w.shape[0]
    A, W = dev_bits(a), dev_bits(w)
    si, sv, parts = _split_router(A, W, n, topk, world)
    oi, ov, full = _one_device(A, W, n, topk)
    for r, p in enumerate(parts):
        b, e = sharded.shard_columns(n, world, r)
        assert np.array_equal(p.view(np.uint32), full[:, b:e].view(np.uint32))
    assert np.array_equal(si, oi)
    assert np.array_equal(sv.view(np.uint32), ov.view(np.uint32))
    want_i, want_v = oracle.topk(full, topk)
    assert np.array_equal(si, want_i)


def test_merge_kernel_special_values_and_empty_entries():
    """+-0, NaN and inf candidates keep their bits; index -1 entries are skipped;
    rows with fewer candidates than topk end in (-1, NaN)."""
    vals = np.array([[[0.0, -0.0, 1.0, np.nan], [np.inf, -0.0, 0.0, 1.0]],
                     [[2.0, np.nan, -np.inf, 3.0], [5.0, 5.0, 0.0, 0.0]]], dtype=np.float32)
    idxs = np.array([[[4, 9, 2, 7], [0, 1, -1, 3]],
                     [[10, 11, -1, 13], [14, 15, -1, -1]]], dtype=np.int32)
    cv = torch.from_numpy(vals).cuda()
    ci = torch.from_numpy(idxs).cuda()
    topk = 8
    idx = torch.empty((2, topk), dtype=torch.int32, device="cuda")
    val = torch.empty((2, topk), dtype=torch.float32, device="cuda")
    mr.router_topk_merge(cv, ci, topk, idx, val)
    gi, gv = host(idx), host(val)
    for r in range(2):
        keep = idxs[:, r, :].reshape(-1) >= 0
        cvals = vals[:, r, :].reshape(-1)[keep]
        cids = idxs[:, r, :].reshape(-1)[keep]
        order = np.argsort(cids, kind="stable")        # oracle row laid out by index
        t = min(topk, cvals.size)
        pos, ov = oracle.topk(cvals[order][None, :], t)
        assert np.array_equal(gi[r, :t], cids[order][pos[0]])
        assert np.array_equal(gv[r, :t].view(np.uint32), ov[0].view(np.uint32))
        assert (gi[r, t:] == -1).all() and np.isnan(gv[r, t:]).all()


def test_topk_ex_index_base_and_validation():
    x = torch.randn(3, 700, device="cuda")
    i0 = torch.empty((3, 10), dtype=torch.int32, device="cuda")
    i1 = torch.empty((3, 10), dtype=torch.int32, device="cuda")
    mr.router_topk(x, 10, i0)
    mr.router_topk_ex(x, 10, i1, index_base=12345)
    assert np.array_equal(host(i1), host(i0) + 12345)
    with pytest.raises(mr.MrError):
        mr.router_topk_ex(x, 10, i1, index_base=-1)
    with pytest.raises(mr.MrError):
        mr.router_topk_ex(x, 10, i1, index_base=2 ** 31 - 100)
