"""The five workloads at full size, in the launch configuration the benchmark
times, checked on sampled outputs the oracle can compute one by one.

- routing: the whole batch is routed on the GPU; sampled chunks are re-routed
  by the oracle from the same router inputs (drawn on the GPU, copied back)
- layout: the whole table, bit-exact, for the generator's chunk map
- packing: sampled rows, bit-exact at the addresses the format prescribes
- decode: sampled (sequence, head) pairs against fp64 attention
"""
import numpy as np
import pytest
import torch

from chunk_adaptive_mixed_b200 import workloads as W
from oracle import oracle as O

from .gpu_helpers import (Case, check_attention, check_layout, check_route, dev, gpu_decode,
                          gpu_layout, gpu_pack, gpu_route, oracle_row, packed_row)

pytestmark = pytest.mark.gpu


def _case(w, lens):
    return Case(lens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.chunk_len, w.kv_dtype)


def _chunk_starts(lens, L):
    return np.concatenate([[0], np.cumsum((lens.astype(np.int64) + L - 1) // L)])


@pytest.mark.parametrize("name", list(W.WORKLOAD_ORDER))
def test_route_full_size_sampled(name):
    w = W.get(name)
    lens = W.seq_lens(w)
    case = _case(w, lens)
    W1, W2, W3, b3 = W.router_weights(w, device=dev())
    C = W.router_input(w, lens, device=dev())
    te, ce, logits = gpu_route(case, C, W1, W2, W3, b3)
    del C
    torch.cuda.empty_cache()
    starts = _chunk_starts(lens, w.chunk_len)
    assert np.all(ce[starts[:-1][lens > 0]] == 0)            # routing freezing
    counts = W.chunk_token_counts(lens, w.chunk_len)
    row0 = np.concatenate([[0], np.cumsum(counts)])
    N = len(counts)
    # at least 128 chunks (all of them for smaller batches): groups of 4
    # consecutive chunks spread evenly over the batch, every sequence's first
    # chunk and the batch's last chunk
    ng = 32
    g0 = np.unique(np.linspace(0, max(N - 4, 0), ng).round().astype(np.int64))
    sample = sorted({int(c) for s0 in g0 for c in range(s0, min(s0 + 4, N))}
                    | {int(c) for c in starts[:-1][lens > 0][:16]} | {N - 1})
    W1c, W2c, W3c, b3c = (x.cpu().numpy() for x in (W1, W2, W3, b3))
    first_chunks = set(starts[:-1].tolist())
    near_total = exempt_total = tokens = 0
    for gc in sample:
        Cs = W.router_input(w, lens, device=dev(), chunk_range=(gc, gc + 1)).cpu().numpy()
        z32, z64 = O.router_logits(Cs, W1c, W2c, W3c, b3c)
        r0, r1 = int(row0[gc]), int(row0[gc + 1])
        n = r1 - r0
        near, exempt = check_route(np.array([n], np.int32), w.chunk_len, te[r0:r1],
                                   ce[gc:gc + 1], logits[r0:r1], z32, z64,
                                   freeze=gc in first_chunks)
        near_total += near
        exempt_total += exempt
        tokens += n
    assert len(sample) >= min(N, 128)
    mix = np.bincount(ce, minlength=3) / len(ce)
    print(f"{name}: {len(sample)} chunks ({tokens} tokens) re-routed by the oracle: "
          f"{near_total} near-tie tokens, {exempt_total} exempt chunks, 0 mismatches outside "
          f"the band; chunk mix FP16/INT4/INT2 = {np.round(mix, 3).tolist()} "
          f"(target {list(w.target_mix)})")
    assert np.abs(mix - np.asarray(w.target_mix)).max() < 0.15


@pytest.mark.parametrize("name", list(W.WORKLOAD_ORDER))
def test_pack_decode_full_size_sampled(name):
    w = W.get(name)
    lens = W.seq_lens(w)
    case = _case(w, lens)
    L, d, Hkv, Hq = w.chunk_len, w.head_dim, w.num_kv_heads, w.num_q_heads
    cmap = W.synthetic_chunk_map(lens, L, mix=w.target_mix, seed=1)
    layout = gpu_layout(case, cmap)
    _, pb = check_layout(case, layout.cpu().numpy(), cmap)
    ob, _ = O.build_layout(Hkv, d, L, lens, cmap)
    _, seqs, _, inv = O.parse_layout(ob, case.B)
    cu = W.cu_seqlens(lens)
    rng = np.random.default_rng(5)
    layers = [0] if w.layers == 1 else [0, w.layers - 1]
    steps = [0] if w.decode_steps == 1 else [0, w.decode_steps - 1]
    for layer in layers:
        K, V = W.kv_layer(w, lens, layer, device=dev())
        packed, gpb = gpu_pack(case, layout, K, V)
        assert gpb == pb
        pk = packed.cpu().numpy()
        # sampled rows, bit-exact (tail tokens of each sequence included)
        nonempty = np.nonzero(lens > 0)[0]
        picks = [(b, int(lens[b]) - 1) for b in nonempty[:3]]
        for _ in range(300):
            b = int(rng.choice(nonempty))
            picks.append((b, int(rng.integers(0, lens[b]))))
        for b, t in picks:
            e = int(cmap[seqs[b]["chunk_offset"] + t // L])
            for kv, src in ((0, K), (1, V)):
                g = int(rng.integers(0, Hkv))
                x = src[cu[b] + t, g].float().cpu().numpy()
                want_c, want_s = oracle_row(x, e)
                got_c, got_s = packed_row(pk, seqs, inv, L, Hkv, d, b, t, kv, g, e,
                                          seqs[b]["chunk_offset"])
                assert np.array_equal(got_c, want_c), (name, layer, b, t, kv, g, e)
                if e:
                    assert np.array_equal(got_s, want_s), (name, layer, b, t, kv, g, e)
        # sampled decode outputs
        seq_pick = sorted(set([int(nonempty[0]), int(nonempty[-1])] +
                              rng.choice(nonempty, 2).tolist()))
        for step in steps:
            q = W.query(w, layer, step, device=dev())
            out = gpu_decode(case, layout, packed, q)
            qn = q.cpu().numpy()
            for b in seq_pick:
                Kb = K[cu[b]:cu[b + 1]].cpu().numpy()
                Vb = V[cu[b]:cu[b + 1]].cpu().numpy()
                mb = cmap[seqs[b]["chunk_offset"]: seqs[b]["chunk_offset"] + seqs[b]["num_chunks"]]
                heads = sorted(set([0, Hq - 1] + rng.integers(0, Hq, 2).tolist()))
                pairs = np.array([[0, h] for h in heads], np.int32)
                want = O.decode_pairs(Hq, Hkv, d, L, np.array([lens[b]], np.int32), mb, Kb, Vb,
                                      qn[b:b + 1], pairs)
                check_attention(out[b, heads], want, f"{name} layer {layer} step {step} seq {b}")
        del K, V, packed
        torch.cuda.empty_cache()
