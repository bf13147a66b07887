"""The benchmark's multi-rank plumbing with two gloo ranks on the CPU: the
slowest rank's time sets the step, work adds up over ranks, and every rank
draws a different batch of the same workload (weak scaling, no collective on
the data path).  Each rank runs the oracle on its own shard (a small BLASST
prefill drawn with its seed); the whole job's executed tiles are the sum over
ranks, and every rank's result equals the same shard computed in one
process."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    try:
        _run(rank, world, port, q)
    except BaseException as e:  # report instead of dying silently
        import traceback
        q.put((rank, "error", traceback.format_exc()))


def _run(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        t_max = bench.max_over_ranks(10.0 + rank)            # ms of this rank
        units = bench.sum_over_ranks(100.0 * (rank + 1))
        rate = bench.whole_job_rate(100.0 * (rank + 1), 10.0 + rank)
        seeds = bench.rank_seeds(rank)
        # this rank's shard: the same recipe drawn with its seed, through the oracle
        o_sum, executed = _shard(seeds[0])
        total_executed = bench.sum_over_ranks(float(executed))
        q.put((rank, t_max, units, rate, seeds, o_sum, executed, total_executed))
    finally:
        dist.destroy_process_group()


def _shard(seed):
    """(sum of O, executed tiles) of the oracle on a small causal BLASST
    prefill drawn with `seed` (B1, 2 query / 1 KV heads, 384 tokens, d 64,
    tiles of 64, a = 10)."""
    import math

    import oracle
    from block_sparse_attention_bsattn_b200 import inputs
    N = 384
    q, k, v = inputs.blasst_prefill_qkv(1, 2, 1, N, 64, "cpu", seed)
    r = oracle.prefill(q, k, v, 64, 1 / math.sqrt(64), True, inputs.lambda_for(10, N))
    return float(r["o"].sum()), int((r["status"] == 2).sum())


def test_two_rank_reductions_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(2)), key=lambda x: x[0])
    errs = [r for r in res if r[1] == "error"]
    assert not errs, errs[0][2]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, t0, u0, rate0, s0, o0, e0, tot0), (r1, t1, u1, rate1, s1, o1, e1, tot1) = res
    assert t0 == t1 == 11.0                     # slowest rank
    assert u0 == u1 == 300.0                    # work of both ranks
    assert rate0 == rate1 == pytest.approx(300.0 / 11e-3)
    assert s0 != s1 and o0 != o1                # different batches per rank
    # each rank's shard equals the same shard computed in one process, and
    # the job's executed tiles are the sum of the shards'
    (ro0, re0), (ro1, re1) = _shard(s0[0]), _shard(s1[0])
    assert (o0, e0) == (ro0, re0) and (o1, e1) == (ro1, re1)
    assert tot0 == tot1 == float(re0 + re1)
