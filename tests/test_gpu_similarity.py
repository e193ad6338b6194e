"""Similarity-based chunk search (Cocktail's chunk-level quantization search)
on the GPU against the CPU oracle.

The similarity is compared in fp64 within SIM_TOL; the chunk map must be
identical except for chunks whose oracle similarity lies within SIM_TOL of a
threshold (both sides decide in fp64, summing in different orders)."""
import numpy as np
import pytest
import torch

from chunk_adaptive_mixed_b200 import mqkv as M
from chunk_adaptive_mixed_b200 import workloads as W
from oracle import oracle as O

from .gpu_helpers import (Case, check_attention, check_layout, dev, gpu_decode, gpu_layout,
                          gpu_pack, random_kv)

pytestmark = pytest.mark.gpu

# fp64 sums of at most a few million fp32 terms in another order: the cosine
# moves by far less than this
SIM_TOL = 1e-9


def gpu_similarity(case, C, u, tau_hi, tau_lo, freeze=True):
    ce = torch.full((max(case.N, 16),), 255, dtype=torch.uint8, device=dev())
    sim = torch.full((max(case.N, 2),), float("nan"), dtype=torch.float64, device=dev())
    M.mq_similarity_route(case.shape(), case.lens, case.cu(), C, u, tau_hi, tau_lo, ce, sim,
                          routing_freeze=freeze)
    torch.cuda.synchronize()
    assert M.mq_device_status() == 0
    return ce[:case.N].cpu().numpy(), sim[:case.N].cpu().numpy()


def check_similarity(ce, sim, ce_o, sim_o, tau_hi, tau_lo):
    assert np.all(np.isfinite(sim))
    err = np.abs(sim - sim_o)
    assert err.max(initial=0.0) <= SIM_TOL, f"similarity off by {err.max():.3e}"
    near = (np.abs(sim_o - tau_hi) < SIM_TOL) | (np.abs(sim_o - tau_lo) < SIM_TOL)
    bad = (ce != ce_o) & ~near
    assert not bad.any(), f"{bad.sum()} chunks differ away from a threshold"
    return int(near.sum())


def _inputs(lens, D, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    T = int(np.sum(lens))
    C = torch.randn(T, D, generator=g) * scale
    u = torch.randn(len(lens), D, generator=g)
    return C, u


SMALL = [
    # lens, D, L: several chunks, ragged tails, an empty sequence, D not a
    # multiple of the 1024 columns a CTA covers per pass
    (np.array([1000], np.int32), 256, 64),
    (np.array([300, 0, 65, 1], np.int32), 4, 32),
    (np.array([4096, 777, 128], np.int32), 4100, 128),
    (np.array([5000], np.int32), 512, 4096),
]


@pytest.mark.parametrize("lens,D,L", SMALL)
@pytest.mark.parametrize("freeze", [True, False])
def test_similarity_matches_oracle(lens, D, L, freeze):
    case = Case(lens, 4, 4, 64, L)
    C, u = _inputs(lens, D, seed=D + L)
    # chunk means are N(0, 1/n) per coordinate, so the cosine spreads ~1/sqrt(D)
    tau_hi, tau_lo = 0.5 / np.sqrt(D), -0.3 / np.sqrt(D)
    ce, sim = gpu_similarity(case, C.to(dev()), u.to(dev()), tau_hi, tau_lo, freeze)
    ce_o, sim_o = O.similarity_route(lens, L, C.numpy(), u.numpy(), tau_hi, tau_lo, freeze)
    check_similarity(ce, sim, ce_o, sim_o, tau_hi, tau_lo)
    if case.N >= 8:
        assert len(set(ce.tolist())) >= 2


def test_similarity_special_cases():
    # zero query (sequence 1), an all-zero chunk (sequence 0, chunk 1), chunks
    # that are exact multiples of the query (cos = +1 and -1), large values
    L, D = 32, 64
    lens = np.array([4 * L, 2 * L, 3 * L + 5], np.int32)
    case = Case(lens, 4, 4, 64, L)
    C, u = _inputs(lens, D, seed=7)
    u[1] = 0.0
    C[L:2 * L] = 0.0
    C[2 * L:3 * L] = 3.0 * u[0]
    C[3 * L:4 * L] = -1e30 * u[0]
    for tau_hi, tau_lo in [(0.5, -0.5), (1.0, -1.0), (0.0, 0.0), (-2.0, 2.0)]:
        ce, sim = gpu_similarity(case, C.to(dev()), u.to(dev()), tau_hi, tau_lo, freeze=False)
        ce_o, sim_o = O.similarity_route(lens, L, C.numpy(), u.numpy(), tau_hi, tau_lo, False)
        check_similarity(ce, sim, ce_o, sim_o, tau_hi, tau_lo)
        assert sim[1] == 0.0 and np.all(sim[4:6] == 0.0)        # zero chunk, zero query
        assert abs(sim[2] - 1.0) < 1e-12 and abs(sim[3] + 1.0) < 1e-12


@pytest.mark.parametrize("name", list(W.WORKLOAD_ORDER))
def test_similarity_full_size_sampled(name):
    """The whole batch is searched on the GPU in the benchmark's configuration;
    sampled chunks are re-scored by the oracle from the same inputs (drawn on
    the GPU by the seeded generator and copied back)."""
    w = W.get(name)
    lens = W.seq_lens(w)
    case = Case(lens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.chunk_len, w.kv_dtype)
    C = W.router_input(w, lens, device=dev())
    u = W.similarity_query(w, device=dev())
    tau_hi, tau_lo = W.similarity_thresholds(w)
    ce, sim = gpu_similarity(case, C, u, tau_hi, tau_lo)
    del C
    torch.cuda.empty_cache()
    L = w.chunk_len
    starts = np.concatenate([[0], np.cumsum((lens.astype(np.int64) + L - 1) // L)])
    assert np.all(ce[starts[:-1][lens > 0]] == 0)               # routing freezing
    seq_of = np.repeat(np.arange(len(lens)), np.diff(starts))
    counts = W.chunk_token_counts(lens, L)
    N = len(counts)
    rng = np.random.default_rng(1)
    sample = sorted(set([0, 1, N // 2, N - 1, int(starts[-2])] + rng.integers(0, N, 6).tolist()))
    un = u.cpu().numpy()
    for gc in sample:
        Cs = W.router_input(w, lens, device=dev(), chunk_range=(gc, gc + 1)).cpu().numpy()
        b = int(seq_of[gc])
        first = gc == starts[b]
        ce_o, sim_o = O.similarity_route(np.array([counts[gc]], np.int32), L, Cs, un[b:b + 1],
                                         tau_hi, tau_lo, routing_freeze=first)
        check_similarity(ce[gc:gc + 1], sim[gc:gc + 1], ce_o, sim_o, tau_hi, tau_lo)
    mix = np.bincount(ce, minlength=3) / N
    print(f"{name}: similarity mix {np.round(mix, 3).tolist()} (target {list(w.target_mix)})")
    if N >= 256:
        assert np.abs(mix - np.asarray(w.target_mix)).max() < 0.1


def test_similarity_map_drives_the_whole_path():
    """Similarity map -> layout -> pack -> decode, each against the oracle."""
    w = W.get("tiny")
    lens = np.array([1000, 64, 333], np.int32)
    case = Case(lens, 8, 4, 64, w.chunk_len, "f16")
    C, u = _inputs(lens, 256, seed=3)
    tau_hi, tau_lo = 0.5 / 16, -0.3 / 16
    ce, sim = gpu_similarity(case, C.to(dev()), u.to(dev()), tau_hi, tau_lo)
    ce_o, sim_o = O.similarity_route(lens, case.L, C.numpy(), u.numpy(), tau_hi, tau_lo)
    assert check_similarity(ce, sim, ce_o, sim_o, tau_hi, tau_lo) == 0
    assert np.array_equal(ce, ce_o)
    layout = gpu_layout(case, ce)
    check_layout(case, layout.cpu().numpy(), ce_o)
    K, V, q = random_kv(case, seed=11)
    packed, pb = gpu_pack(case, layout, K.to(dev()), V.to(dev()))
    ref = O.pack(case.Hkv, case.d, case.L, lens, ce_o, K.numpy(), V.numpy())
    assert np.array_equal(packed[:pb].cpu().numpy(), ref)
    out = gpu_decode(case, layout, packed, q.to(dev()))
    want = O.decode(case.Hq, case.Hkv, case.d, case.L, lens, ce_o, ref, q.numpy())
    check_attention(out, want, "similarity map")
