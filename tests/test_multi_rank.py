"""The multi-GPU path of the benchmark on CPU: two gloo ranks.

The path shards by batch: every rank routes, packs and decodes its own
sequences, with no data-path exchange.  What the ranks share is the timing:
a barrier around the timed region and the max over ranks of the elapsed
time.  These tests run that plumbing with gloo on 127.0.0.1."""
import os
import socket

import pytest
import torch.distributed as tdist
import torch.multiprocessing as mp

import bench
from chunk_adaptive_mixed_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.get("llama3_8b_gqa")
        seed = bench.rank_seed(0, rank)
        lens = W.seq_lens(w, seed)
        q = W.query(w, 0, 0, seed)
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        tdist.barrier()
        ms = bench.reduce_timing(local_ms)
        value = bench.job_throughput(len(lens) * w.decode_steps, world, ms)
        # the end-to-end entry: bytes summed over ranks, the slowest time
        e2e = bench.e2e_result(len(lens) * w.decode_steps, world, ms,
                               bench.reduce_sum(1000.0 + rank), bench.reduce_sum(10.0 * (rank + 1)),
                               3, False)
        out[rank] = (int(lens.sum()), float(q.float().sum()), ms, value, e2e)
    finally:
        tdist.destroy_process_group()


def test_two_gloo_ranks_shard_batches_and_take_the_max_time():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    (t0, q0, ms0, v0, e0), (t1, q1, ms1, v1, e1) = res[0], res[1]
    assert ms0 == ms1 == 15.0                    # the slowest rank's time on both
    assert v0 == v1 == pytest.approx(64 * 100 * 2 / 0.015)
    assert (t0, q0) != (t1, q1)                  # each rank drew its own batch
    assert e0 == e1
    assert e0["value"] == pytest.approx(v0) and e0["ms_per_step"] == 15.0
    assert (e0["h2d_bytes_per_step"], e0["d2h_bytes_per_step"]) == (2001, 30)


def test_single_process_timing_is_local():
    assert bench.reduce_timing(3.5) == 3.5
    assert bench.reduce_sum(7.0) == 7.0
    assert bench.job_throughput(4, 1, 20.0) == pytest.approx(200.0)
    e = bench.e2e_result(4, 1, 20.0, 100, 8, 2, False)
    assert e["value"] == pytest.approx(200.0)
    assert (e["h2d_bytes_per_step"], e["d2h_bytes_per_step"], e["steps"]) == (100, 8, 2)
    # a split context: every rank decodes the same sequences
    assert bench.e2e_result(4, 2, 20.0, 100, 8, 2, True)["value"] == pytest.approx(200.0)
