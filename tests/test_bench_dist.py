"""The bench's multi-rank logic on CPU (gloo, world size 2): max-over-ranks
timing, barriers, and rank 0 alone printing the reference arm."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        w, r, lr = bench.dist_env()

        class Args:
            steps, warmup = 1, 0
        ref = bench.run_reference(Args, world, rank, budget_s=2.0) if rank == 1 else None
        q.put((rank, t, (w, r, lr), ref))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_is_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [15.0, 15.0]
    assert [o[2] for o in out] == [(2, 0, 0), (2, 1, 1)]
    assert out[1][3] is None  # only rank 0 runs and prints the reference arm


def test_source_hash_ignores_comments_only():
    """A recorded ncu traffic figure stays valid across comment edits and is
    dropped by any code edit."""
    import bench
    code = "int f(int x) {\n    return x + 1;  // one\n}\n/* block\n comment */\n"
    assert bench._code_only(code) == bench._code_only(code.replace("// one", "// two").replace("block", "other"))
    assert bench._code_only(code) != bench._code_only(code.replace("x + 1", "x + 2"))
