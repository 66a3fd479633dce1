"""The multi-rank host path of bench.py on CPU: two gloo ranks, one process
each.  Every rank runs its own batch (replicas), the step time is the max over
ranks, and the whole-job rate counts all ranks' FLOPs.  Also checks that the
per-rank inputs differ (each rank draws its own seeded batch) and that a rank
which raises is reported to the launcher rather than hanging the other.

The bias gradients (a T5 table's, the ALiBi slopes') are weight gradients:
each replica's covers its own batch shard, and the training framework's
weight-gradient all-reduce sums them.  The last test checks, with the
oracle on two gloo ranks, that the sum of the shards' gradients is the
gradient of the whole batch."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out, fail_rank):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import bench
    from scaled_dot_product_bwd_b200.inputs import make_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        if rank == fail_rank:
            raise RuntimeError("rank failed before its step")
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms)
        q = make_inputs(1, 16, 2, 1, 64, seed=rank).q
        gathered = [torch.empty_like(q.float()) for _ in range(world)]
        dist.all_gather(gathered, q.float())
        out[rank] = (slowest, bench.whole_job_tflops(world, 10**12, slowest),
                     bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


def _run(fail_rank=-1):
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out, fail_rank)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    return dict(out), codes


def test_two_gloo_ranks_max_time_and_weak_scaling():
    out, codes = _run()
    assert codes == [0, 0], codes
    for r in range(2):
        slowest, tflops, same = out[r]
        assert slowest == 15.0                       # max over ranks
        assert tflops == pytest.approx(2 * 1e12 / 15e-3 / 1e12)
        assert not same                              # each rank has its own batch


def test_failing_rank_is_reported_not_hung():
    out, codes = _run(fail_rank=1)
    assert codes[1] != 0                             # the failing rank exits non-zero
    assert all(c is not None for c in codes)         # nobody is left hanging


def _grad_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    from oracle import alibi_slope_gradient, attention_backward, t5_table_gradient
    from scaled_dot_product_bwd_b200.inputs import make_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        full = make_inputs(2 * world, 24, 2, 1, 8, seed=5, t5_buckets=8, alibi=True)
        sl = slice(2 * rank, 2 * rank + 2)            # this rank's batch shard
        args = (full.q[sl], full.k[sl], full.v[sl], full.do[sl])
        *_, dS = attention_backward(*args, causal=True, t5_table=full.t5_table,
                                    t5_num_buckets=8, t5_max_distance=12, return_dbias=True)
        table = torch.from_numpy(t5_table_gradient(dS, 8, 12, True))
        *_, dS2 = attention_backward(*args, causal=True, alibi_slopes=full.alibi_slopes,
                                     return_dbias=True)
        slopes = torch.from_numpy(alibi_slope_gradient(dS2))
        dist.all_reduce(table)
        dist.all_reduce(slopes)
        out[rank] = (table.numpy(), slopes.numpy())
    finally:
        dist.destroy_process_group()


def test_bias_gradients_of_batch_shards_sum_to_the_full_batch():
    import numpy as np

    from oracle import alibi_slope_gradient, attention_backward, t5_table_gradient
    from scaled_dot_product_bwd_b200.inputs import make_inputs
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_grad_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert [p.exitcode for p in procs] == [0, 0]
    full = make_inputs(2 * world, 24, 2, 1, 8, seed=5, t5_buckets=8, alibi=True)
    args = (full.q, full.k, full.v, full.do)
    *_, dS = attention_backward(*args, causal=True, t5_table=full.t5_table, t5_num_buckets=8,
                                t5_max_distance=12, return_dbias=True)
    *_, dS2 = attention_backward(*args, causal=True, alibi_slopes=full.alibi_slopes,
                                 return_dbias=True)
    want_table = t5_table_gradient(dS, 8, 12, True)
    want_slopes = alibi_slope_gradient(dS2)
    for r in range(world):
        assert np.allclose(out[r][0], want_table, atol=1e-12)
        assert np.allclose(out[r][1], want_slopes, atol=1e-10)
