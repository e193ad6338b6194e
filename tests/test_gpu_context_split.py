"""A batch split by context, on one GPU: the shards of W ranks are decoded one
after another (separate launches that never wait on each other), their
records stacked as an all-gather would, and merged by mq_combine_partials.
Checked against the CPU oracle: every shard's records, and the merged output
against attention over the whole sequences.  The router, run on each shard
with freezing only on shard 0, must reproduce the whole-batch map."""
import numpy as np
import pytest
import torch

from chunk_adaptive_mixed_b200 import context_split as CS
from chunk_adaptive_mixed_b200 import mqkv as M
from chunk_adaptive_mixed_b200 import workloads as W
from oracle import oracle as O

from .gpu_helpers import (REL_L2, Case, check_attention, dev, gpu_layout, gpu_pack, gpu_route,
                          random_kv)

pytestmark = pytest.mark.gpu

LSE_TOL = REL_L2 / 2


def _gpu_records(case, layout, packed, q):
    rec = torch.full((case.B, case.Hq, case.d + 4), float("nan"), dtype=torch.float32,
                     device=dev())
    ws = torch.empty(M.mq_decode_workspace_bytes(case.shape(), case.lens), dtype=torch.uint8,
                     device=dev())
    M.mq_decode_attn_partial(case.shape(), case.lens, layout, packed, q, rec, ws)
    torch.cuda.synchronize()
    assert M.mq_device_status() == 0
    return rec


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("d,L,hq,hkv,dtype", [(128, 64, 8, 2, "f16"), (64, 32, 4, 4, "f32")])
def test_context_split_records_merge_to_whole_attention(world, d, L, hq, hkv, dtype):
    lens = np.array([900, 96, 0, 31, 260], np.int32)
    full = Case(lens, hq, hkv, d, L, dtype)
    K, V, q = random_kv(full, seed=world + d)
    cmap = W.synthetic_chunk_map(lens, L, mix=(0.2, 0.5, 0.3), seed=world)
    recs = []
    for r in range(world):
        lo, hi = CS.shard_ranges(lens, L, r, world)
        case = Case(CS.shard_lengths(lens, L, r, world), hq, hkv, d, L, dtype)
        m = CS.shard_chunk_map(cmap, lens, L, r, world)
        Ks, Vs = CS.shard_rows(K, lens, lo, hi), CS.shard_rows(V, lens, lo, hi)
        layout = gpu_layout(case, m)
        packed, _ = gpu_pack(case, layout, Ks.to(dev()), Vs.to(dev()))
        rec = _gpu_records(case, layout, packed, q.to(dev()))
        # this shard's records against the oracle's
        ref = O.pack(hkv, d, L, case.lens, m, Ks.numpy(), Vs.numpy())
        o, ml = O.decode_partial(hq, hkv, d, L, case.lens, m, ref, q.numpy())
        got = rec.cpu().numpy().astype(np.float64)
        check_attention(got[..., :d], o, f"shard {r} output")
        empty = ml[..., 1] == 0
        assert np.all(got[..., d][empty] == -np.inf) and np.all(got[..., d + 1][empty] == 0)
        # m is a reference score (the decode rescales lazily), so only the
        # log-sum-exp m + log l of the shard's scores is fixed.  An error e in
        # it scales the shard's weight in the merge by about 1 + e, moving the
        # merged output by at most ~e |o|: LSE_TOL = REL_L2 / 2 keeps the merge
        # inside the attention tolerance (observed: ~5e-5 with fp16 queries,
        # ~4e-4 with fp32 queries, whose products with the codes are rounded)
        lse_g = got[..., d][~empty] + np.log(got[..., d + 1][~empty])
        lse_o = ml[..., 0][~empty] + np.log(ml[..., 1][~empty])
        assert np.allclose(lse_g, lse_o, rtol=0, atol=LSE_TOL), np.abs(lse_g - lse_o).max()
        assert np.all(got[..., d][~empty] >= ml[..., 0][~empty] - 8 * np.log(2) - 1e-4)
        recs.append(rec)
    stacked = torch.stack(recs)
    out = torch.full((full.B, hq, d), float("nan"), dtype=torch.float32, device=dev())
    M.mq_combine_partials(stacked, out)
    torch.cuda.synchronize()
    ref = O.pack(hkv, d, L, lens, cmap, K.numpy(), V.numpy())
    want = O.decode(hq, hkv, d, L, lens, cmap, ref, q.numpy())
    check_attention(out.cpu().numpy(), want, f"merged, world {world}")
    assert np.all(out.cpu().numpy()[lens == 0] == 0.0)


def test_shard_routing_reproduces_the_whole_batch_map():
    w = W.get("tiny")
    lens = np.array([1000, 64, 0, 333], np.int32)
    full = Case(lens, 4, 4, 64, w.chunk_len)
    C = W.router_input(w, lens)
    W1, W2, W3, b3 = (x.to(dev()) for x in W.router_weights(w))
    _, ce_full, _ = gpu_route(full, C.to(dev()), W1, W2, W3, b3, freeze=True)
    world = 3
    for r in range(world):
        lo, hi = CS.shard_ranges(lens, w.chunk_len, r, world)
        case = Case(CS.shard_lengths(lens, w.chunk_len, r, world), 4, 4, 64, w.chunk_len)
        Cs = CS.shard_rows(C, lens, lo, hi)
        _, ce, _ = gpu_route(case, Cs.to(dev()), W1, W2, W3, b3, freeze=CS.routing_freeze(r))
        assert np.array_equal(ce, CS.shard_chunk_map(ce_full, lens, w.chunk_len, r, world)), r


def test_combine_of_one_part_is_the_decode_output():
    case = Case(np.array([500, 0, 77], np.int32), 8, 4, 128, 64, "f16")
    K, V, q = random_kv(case, seed=9)
    cmap = W.synthetic_chunk_map(case.lens, case.L, seed=9)
    layout = gpu_layout(case, cmap)
    packed, _ = gpu_pack(case, layout, K.to(dev()), V.to(dev()))
    rec = _gpu_records(case, layout, packed, q.to(dev()))
    out = torch.empty(case.B, case.Hq, case.d, dtype=torch.float32, device=dev())
    M.mq_combine_partials(rec.unsqueeze(0), out)
    ws = torch.empty(M.mq_decode_workspace_bytes(case.shape(), case.lens), dtype=torch.uint8,
                     device=dev())
    direct = torch.empty_like(out)
    M.mq_decode_attn(case.shape(), case.lens, layout, packed, q.to(dev()), direct, ws)
    torch.cuda.synchronize()
    assert torch.allclose(out, direct, rtol=1e-6, atol=1e-7)
