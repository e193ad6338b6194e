"""A batch split by context across ranks, on CPU: the shard plan, routing with
freezing on the right rank, and the all-gather of records over gloo (world
sizes 2 and 3).  Each rank computes its shard's records with the CPU oracle;
the gathered records, merged with the split-softmax rule, must give the
attention over the whole sequences, and the shard maps must be the slices of
the whole-batch map."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp

from chunk_adaptive_mixed_b200 import context_split as CS
from oracle import oracle as O

LENS = np.array([700, 96, 0, 31, 200], np.int32)   # chunks 11, 2, 0, 1, 4 at L = 64
L, HKV, HQ, D, DR, H = 64, 2, 4, 64, 64, 64


def test_shard_plan_covers_every_token_once():
    for world in (1, 2, 3, 8):
        seen = np.zeros(int(LENS.sum()), np.int32)
        starts = np.concatenate([[0], np.cumsum(LENS)])
        for r in range(world):
            lo, hi = CS.shard_ranges(LENS, L, r, world)
            assert np.all(lo % L == 0) and np.all((hi % L == 0) | (hi == LENS))
            for b in range(len(LENS)):
                seen[starts[b] + lo[b]:starts[b] + hi[b]] += 1
        assert np.all(seen == 1)
    assert CS.routing_freeze(0) and not CS.routing_freeze(1)


def _inputs():
    g = torch.Generator().manual_seed(3)
    T = int(LENS.sum())
    C = torch.randn(T, DR, generator=g)
    K = torch.randn(T, HKV, D, generator=g)
    V = torch.randn(T, HKV, D, generator=g)
    q = torch.randn(len(LENS), HQ, D, generator=g)
    W1 = torch.randn(DR, H, generator=g) / DR ** 0.5
    W2 = torch.randn(DR, H, generator=g) / DR ** 0.5
    W3 = torch.randn(H, 3, generator=g) / H ** 0.5
    return C.numpy(), K.numpy(), V.numpy(), q.numpy(), W1.numpy(), W2.numpy(), W3.numpy()


def _records(lens, cmap, K, V, q):
    ref = O.pack(HKV, D, L, lens, cmap, K, V)
    o, ml = O.decode_partial(HQ, HKV, D, L, lens, cmap, ref, q)
    rec = np.zeros((len(lens), HQ, D + 4), np.float32)
    rec[..., :D] = o
    rec[..., D:D + 2] = ml
    return rec


def _merge(recs):
    m, l = recs[..., D].astype(np.float64), recs[..., D + 1].astype(np.float64)
    M = np.where(l > 0, m, -np.inf).max(axis=0)
    w = np.where(l > 0, l * np.exp(np.where(l > 0, m, 0.0) - np.where(np.isfinite(M), M, 0.0)), 0)
    num = (w[..., None] * recs[..., :D]).sum(axis=0)
    den = w.sum(axis=0)
    return np.where(den[..., None] > 0, num / np.where(den > 0, den, 1)[..., None], 0.0)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        C, K, V, q, W1, W2, W3 = _inputs()
        lo, hi = CS.shard_ranges(LENS, L, rank, world)
        lens = CS.shard_lengths(LENS, L, rank, world)
        Cs, Ks, Vs = (CS.shard_rows(x, LENS, lo, hi) for x in (C, K, V))
        cmap, _, _, _ = O.route(lens, L, Cs, W1, W2, W3, routing_freeze=CS.routing_freeze(rank))
        full_map, _, _, _ = O.route(LENS, L, C, W1, W2, W3, routing_freeze=True)
        maps_ok = np.array_equal(cmap, CS.shard_chunk_map(full_map, LENS, L, rank, world))
        rec = torch.from_numpy(_records(lens, cmap, Ks, Vs, q))
        gathered = CS.gather_records(rec).numpy()
        merged = _merge(gathered)
        ref = O.pack(HKV, D, L, LENS, full_map, K, V)
        want = O.decode(HQ, HKV, D, L, LENS, full_map, ref, q)
        err = float(np.abs(merged - want).max())
        out[rank] = (maps_ok, err, gathered.shape)
    finally:
        tdist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_gather_records_that_merge_to_whole_attention(world):
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        maps_ok, err, shape = res[r]
        assert maps_ok, f"rank {r}: shard map differs from the whole-batch map"
        assert shape == (world, len(LENS), HQ, D + 4)
        assert err < 1e-5, f"rank {r}: merged records off by {err}"  # fp32 records
