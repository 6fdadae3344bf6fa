"""The column-split router's host logic on CPU ranks (gloo, world size 2 and 3).

Each rank owns a contiguous block of the router weight's columns
(``sharded.shard_columns``), computes its shard's logits and top-k with global
indices, and the ranks exchange candidate lists through
``sharded.gather_candidates`` (the same all-gather the GPU path runs over
NCCL).  The merge of the gathered lists must equal the top-k of the full row
bit for bit, with ties across a shard boundary going to the lower index.
Here the oracle computes the shard logits and stands in for the merge kernel
(its top-k over the rank-major candidate list, whose position order is the
index order); the kernel itself is checked on the GPU in test_sharded_gpu.py.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cases():
    """(name, A bits, Wt bits, topk): the router shape, and tie-heavy integer rows."""
    a, w = synth.router(16)
    ties_a = synth.choice_bits(41, (6, 64), "bf16", [-1, 0, 1])
    ties_w = synth.choice_bits(42, (40, 64), "bf16", [-1, 0, 1])
    # Duplicate columns across every possible boundary of 40 columns into 2
    # or 3 shards (19|20 and 12|13, 25|26): bitwise-equal logits on both sides.
    for lo in (19, 12, 25):
        ties_w[lo + 1] = ties_w[lo]
    small_w = synth.choice_bits(43, (7, 64), "bf16", [-2, 0, 2])   # shards narrower than topk
    return [("router", a, w, 10), ("ties", ties_a, ties_w, 10), ("narrow_shards", ties_a, small_w, 5)]


def _merge_with_oracle(cand_val, cand_idx, topk):
    """Top-k of each row's gathered candidates (rank-major order), mapped to global indices."""
    world, m, per = cand_val.shape
    out_i = np.full((m, topk), -1, dtype=np.int32)
    out_v = np.full((m, topk), np.nan, dtype=np.float32)
    for r in range(m):
        vals = cand_val[:, r, :].reshape(-1)
        idx = cand_idx[:, r, :].reshape(-1)
        keep = idx >= 0
        vals, idx = vals[keep], idx[keep]
        t = min(topk, vals.size)
        pos, v = oracle.topk(vals[None, :], t)
        out_i[r, :t] = idx[pos[0]]
        out_v[r, :t] = v[0]
    return out_i, out_v


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from verify_weight_streaming_b200 import sharded
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        results = []
        for name, a, w, topk in _cases():
            n = w.shape[0]
            b, e = sharded.shard_columns(n, world, rank)
            logits, _ = oracle.matmul(a, "bf16", w[b:e], "bf16")
            logits = logits.astype(np.float32)
            k_loc = sharded.local_topk(e - b, topk)
            li, lv = oracle.topk(logits, k_loc)
            m = a.shape[0]
            mine_i = torch.full((m, topk), -1, dtype=torch.int32)
            mine_v = torch.zeros((m, topk), dtype=torch.float32)
            mine_i[:, :k_loc] = torch.from_numpy(li + b)
            mine_v[:, :k_loc] = torch.from_numpy(lv)
            all_i = torch.empty((world, 16, topk), dtype=torch.int32)
            all_v = torch.empty((world, 16, topk), dtype=torch.float32)
            ci, cv = sharded.gather_candidates(mine_i, mine_v, all_i, all_v, world)
            results.append((name, ci.numpy().copy(), cv.numpy().copy(), (b, e)))
        q.put((rank, results))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_column_split_merge_equals_single_device_topk(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for ci_case, (name, a, w, topk) in enumerate(_cases()):
        n = w.shape[0]
        # the shards cover every column once, in rank order
        bounds = [got[r][ci_case][3] for r in range(world)]
        assert bounds[0][0] == 0 and bounds[-1][1] == n
        assert all(bounds[r][1] == bounds[r + 1][0] for r in range(world - 1))
        # every rank gathered the same candidate lists
        for r in range(1, world):
            assert np.array_equal(got[r][ci_case][1], got[0][ci_case][1])
            assert np.array_equal(got[r][ci_case][2].view(np.uint32), got[0][ci_case][2].view(np.uint32))
        _, cand_i, cand_v, _ = got[0][ci_case]
        full, _ = oracle.matmul(a, "bf16", w, "bf16")
        full = full.astype(np.float32)
        want_i, want_v = oracle.topk(full, topk)
        mi, mv = _merge_with_oracle(cand_v, cand_i, topk)
        assert np.array_equal(mi, want_i), (name, world)
        assert np.array_equal(mv.view(np.uint32), want_v.view(np.uint32)), (name, world)


def test_planted_boundary_tie_goes_to_the_lower_index():
    """The tie case really straddles the boundary and reaches the top-k."""
    from verify_weight_streaming_b200 import sharded
    _, a, w, topk = _cases()[1]
    full, _ = oracle.matmul(a, "bf16", w, "bf16")
    assert sharded.shard_columns(40, 2, 0) == (0, 20)
    assert np.array_equal(full[:, 19], full[:, 20])
    idx, _ = oracle.topk(full.astype(np.float32), topk)
    hit = [r for r in range(a.shape[0]) if 19 in idx[r]]
    assert hit, "the planted tie is in no row's top-k"
    for r in hit:
        row = list(idx[r])
        assert 20 in row and row.index(19) < row.index(20)


def test_shard_columns_rejects_bad_splits():
    from verify_weight_streaming_b200 import sharded
    for args in ((3, 4, 0), (8, 0, 0), (8, 2, 2), (8, 2, -1)):
        with pytest.raises(ValueError):
            sharded.shard_columns(*args)
    assert sharded.local_topk(7, 10) == 7 and sharded.local_topk(256, 10) == 10
