"""Multi-process host logic on CPU (gloo, world size 2): the d_in-sharded norm's
column split and its all-reduce of squared partials, the row-sharded norm's
all-gather, the module split of a grouped call, the bench's cross-rank timing
helpers (barrier, max over ranks), and a rank that fails before a collective.
Each rank is a spawned process; the oracle stands in for the GPU calls (there
is no GPU here)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _module(seed=21, d_out=9, d_in=200, r=5):
    rng = np.random.default_rng(seed)
    W0 = rng.standard_normal((d_out, d_in))
    A = rng.standard_normal((r, d_in)) / np.sqrt(d_in)
    B = 0.3 * rng.standard_normal((d_out, r))
    return W0, A, B


def _sharded_norm(rank, world):
    import oracle
    from dora_adapter_factored_b200.sharded import all_reduce_rows, column_shard
    W0, A, B = _module()
    a, b = column_shard(W0.shape[1], rank, world, align=64)
    sq = torch.from_numpy(oracle.factored_row_norm_sq(W0[:, a:b], A[:, a:b], B, 1.5))
    all_reduce_rows(sq)
    return np.sqrt(np.maximum(sq.numpy(), 0.0))


def _row_sharded_norm(rank, world):
    import oracle
    from dora_adapter_factored_b200.sharded import all_gather_rows, row_shard
    W0, A, B = _module(d_out=37)
    a, b = row_shard(37, rank, world, align=8)
    n_local = torch.from_numpy(oracle.dense_row_norm(W0[a:b], A, B[a:b], 1.5))
    return all_gather_rows(n_local, 37, align=8).numpy()


def _bench_helpers(rank, world):
    import bench
    bench.barrier(dist, 0)
    worst = bench.max_over_ranks(dist, float(10 * (rank + 1)))
    bench.barrier(dist, 0)
    return worst


def _failing_rank(rank, world):
    # Rank 1 raises before the collective; rank 0's all-reduce must end with
    # an error at the process group's timeout, not hang.
    if rank == 1:
        raise RuntimeError("planted failure on rank 1")
    t = torch.ones(4)
    try:
        dist.all_reduce(t)
    except Exception as e:  # noqa: BLE001 - any error ends the wait
        return f"error: {type(e).__name__}"
    return "completed"


FNS = {"sharded_norm": _sharded_norm, "row_sharded_norm": _row_sharded_norm,
       "bench_helpers": _bench_helpers, "failing_rank": _failing_rank}


def _worker(rank, world, port, name, timeout_s, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    import sys
    if root not in sys.path:
        sys.path.insert(0, root)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))
    try:
        q.put((rank, "ok", FNS[name](rank, world)))
    except Exception as e:  # noqa: BLE001
        q.put((rank, "raised", repr(e)))
    finally:
        try:
            dist.destroy_process_group()
        except Exception:  # noqa: BLE001
            pass


def _run(name, timeout_s=60):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, WORLD, port, name, timeout_s, q))
             for r in range(WORLD)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(WORLD):
        rank, status, val = q.get(timeout=timeout_s + 60)
        out[rank] = (status, val)
    for p in procs:
        p.join(timeout=30)
        if p.is_alive():
            p.kill()
    return out


def test_column_shards_partition_d_in():
    from dora_adapter_factored_b200.sharded import column_shard
    for d_in in (1, 8, 63, 64, 200, 1000, 8192, 25600):
        for world in (1, 2, 3, 4, 8):
            bounds = [column_shard(d_in, r, world) for r in range(world)]
            assert bounds[0][0] == 0 and bounds[-1][1] == d_in
            for (a0, b0), (a1, b1) in zip(bounds, bounds[1:]):
                assert b0 == a1
            for a, b in bounds:
                assert a <= b and (a % 64 == 0 or a == d_in)
    with pytest.raises(ValueError):
        column_shard(64, 2, 2)


def test_sharded_norm_all_reduce_two_ranks():
    import oracle
    out = _run("sharded_norm")
    W0, A, B = _module()
    dense = oracle.dense_row_norm(W0, A, B, 1.5)
    for rank in range(WORLD):
        status, n = out[rank]
        assert status == "ok", n
        np.testing.assert_allclose(n, dense, rtol=1e-12)


def test_row_sharded_norm_all_gather_two_ranks():
    import oracle
    out = _run("row_sharded_norm")
    W0, A, B = _module(d_out=37)
    dense = oracle.dense_row_norm(W0, A, B, 1.5)
    for rank in range(WORLD):
        status, n = out[rank]
        assert status == "ok", n
        np.testing.assert_array_equal(n, dense)


def test_module_shard_balances_and_covers():
    from dora_adapter_factored_b200.sharded import module_shard
    rng = np.random.default_rng(5)
    for world in (1, 2, 3, 8):
        flops = list(rng.uniform(1, 10, 56))
        parts = module_shard(flops, world)
        assert sorted(i for p in parts for i in p) == list(range(56))
        assert all(p == sorted(p) for p in parts)
        loads = [sum(flops[i] for i in p) for p in parts]
        assert max(loads) <= sum(flops) / world + max(flops) + 1e-9
        assert module_shard(flops, world) == parts  # deterministic
    # a decoder layer's seven modules on three ranks: each gets a share
    layer = [2 * 4096 * 4096, 2 * 1024 * 4096, 2 * 1024 * 4096, 2 * 4096 * 4096,
             2 * 14336 * 4096, 2 * 14336 * 4096, 2 * 4096 * 14336]
    assert all(module_shard(layer, 3))


def test_bench_rank_helpers_two_ranks():
    out = _run("bench_helpers")
    for rank in range(WORLD):
        assert out[rank] == ("ok", 10.0 * WORLD)


def test_a_failing_rank_ends_the_others_wait():
    out = _run("failing_rank", timeout_s=5)
    assert out[1][0] == "raised"
    assert out[0][0] == "ok" and out[0][1].startswith("error"), out[0]
