"""Seeded synthetic workloads for the mixed-bitwidth KV-cache path.

This module only draws random inputs; it holds none of the method's
arithmetic.  Both the CUDA path and the CPU oracle take their inputs from
here.  Tensors are drawn with torch generators on the requested device, so a
caller that needs the same values on both sides draws once and copies.

The shapes follow the models named in each workload (no checkpoints or
datasets exist here: every tensor is random, of that model's shape):

  tiny              1 layer, 1 x 1024 tokens, 4 heads x 64, chunk 64, D=256, H=64,
                    fp32; key channels 3 and 40 x8; ~20/50/30 FP16/INT4/INT2
  llama2_7b_layer   1 layer, 1 x 4096 tokens, 32 heads x 128, chunk 128, D=4096,
                    H=256, fp16; 4 seeded key channels x10, token-0 key x5;
                    ~15/60/25
  llama2_7b_32l     32 layers sharing one routing map, 4 x 32768 tokens, same
                    shape and distribution as llama2_7b_layer, K/V of layer l
                    drawn from seed + l
  llama2_13b_128k   40 layers, 1 x 131072 tokens, 40 heads x 128, chunk 256,
                    D=5120, H=256, fp16; ~5/35/60; K/V drawn and packed one
                    layer at a time, only the packed cache resident
  llama3_8b_gqa     1 layer, 64 sequences of lengths uniform in [2048, 16384],
                    32 query / 8 KV heads x 128, chunk 128, D=4096, H=256, fp16;
                    ~15/60/25; a fresh fp16 query per decode step, 100 steps

Router input C: tokens of one chunk share a common direction,
C_t = sqrt(rho) * z_chunk + sqrt(1 - rho) * z_t with z ~ N(0, I) and rho = 0.9,
so each coordinate is N(0, 1) and chunks differ from one another (with
independent tokens every chunk would vote alike).  W1, W2 ~ N(0, 1/D),
W3 ~ N(0, 1/H).  The similarity search takes one query vector per sequence,
u_b ~ N(0, I), independent of C; the cosine of two independent directions in
D dimensions is close to N(0, 1/D), so its thresholds are that normal's
quantiles at the target mix.  The per-expert bias b3 of each workload is a fixed input that
was chosen offline with the CPU oracle (tests/golden/fit_router_bias.py) so
that the chunk-level mix lands near the target; the achieved mix is measured
and reported, never assumed.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import numpy as np
import torch

EXPERT_NAMES = ("FP16", "INT4", "INT2")
EXPERT_BITS = (16, 4, 2)

# stream tags for seed derivation
_TAG = {"seq_lens": 1, "c_chunk": 2, "c_token": 3, "w1": 4, "w2": 5, "w3": 6, "k": 7, "v": 8,
        "q": 9, "outliers": 10, "map": 11, "u": 12, "k_new": 13, "v_new": 14, "c_new": 15}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    layers: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    chunk_len: int
    router_dim: int
    router_hidden: int
    kv_dtype: str                      # "f32" or "f16"; q and C follow (C is always fp32)
    seq_len: Optional[int]             # fixed length, or
    seq_len_range: Optional[Tuple[int, int]]  # inclusive uniform range
    target_mix: Tuple[float, float, float]
    router_bias: Tuple[float, float, float]
    outlier_channels: Optional[Tuple[int, ...]]  # fixed channels, or None = seeded
    num_outlier_channels: int
    outlier_scale: float
    sink_scale: float                  # token 0's key is multiplied by this
    decode_steps: int = 1
    chunk_corr: float = 0.9
    # K/V drawn and packed one layer at a time (only the packed cache of every
    # layer stays resident), instead of every layer's K/V resident at once
    kv_streamed: bool = False

    @property
    def torch_dtype(self):
        return torch.float32 if self.kv_dtype == "f32" else torch.float16

    @property
    def qpg(self):
        return self.num_q_heads // self.num_kv_heads


WORKLOADS = {
    "tiny": Workload(
        name="tiny", layers=1, num_seqs=1, num_q_heads=4, num_kv_heads=4, head_dim=64,
        chunk_len=64, router_dim=256, router_hidden=64, kv_dtype="f32", seq_len=1024,
        seq_len_range=None, target_mix=(0.20, 0.50, 0.30),
        router_bias=(0.0, -0.05, -0.2),
        outlier_channels=(3, 40), num_outlier_channels=2, outlier_scale=8.0, sink_scale=1.0),
    "llama2_7b_layer": Workload(
        name="llama2_7b_layer", layers=1, num_seqs=1, num_q_heads=32, num_kv_heads=32,
        head_dim=128, chunk_len=128, router_dim=4096, router_hidden=256, kv_dtype="f16",
        seq_len=4096, seq_len_range=None, target_mix=(0.15, 0.60, 0.25),
        router_bias=(0.0, 0.522, 0.176),
        outlier_channels=None, num_outlier_channels=4, outlier_scale=10.0, sink_scale=5.0),
    "llama2_7b_32l": Workload(
        name="llama2_7b_32l", layers=32, num_seqs=4, num_q_heads=32, num_kv_heads=32,
        head_dim=128, chunk_len=128, router_dim=4096, router_hidden=256, kv_dtype="f16",
        seq_len=32768, seq_len_range=None, target_mix=(0.15, 0.60, 0.25),
        router_bias=(0.0, 0.522, 0.176),
        outlier_channels=None, num_outlier_channels=4, outlier_scale=10.0, sink_scale=5.0),
    "llama2_13b_128k": Workload(
        name="llama2_13b_128k", layers=40, num_seqs=1, num_q_heads=40, num_kv_heads=40,
        head_dim=128, chunk_len=256, router_dim=5120, router_hidden=256, kv_dtype="f16",
        seq_len=131072, seq_len_range=None, target_mix=(0.05, 0.35, 0.60),
        router_bias=(0.0, 0.88, 0.94),
        outlier_channels=None, num_outlier_channels=4, outlier_scale=10.0, sink_scale=5.0,
        kv_streamed=True),
    "llama3_8b_gqa": Workload(
        name="llama3_8b_gqa", layers=1, num_seqs=64, num_q_heads=32, num_kv_heads=8,
        head_dim=128, chunk_len=128, router_dim=4096, router_hidden=256, kv_dtype="f16",
        seq_len=None, seq_len_range=(2048, 16384), target_mix=(0.15, 0.60, 0.25),
        router_bias=(0.0, 0.52, 0.14),
        outlier_channels=None, num_outlier_channels=4, outlier_scale=10.0, sink_scale=5.0,
        decode_steps=100),
}

WORKLOAD_ORDER = ("tiny", "llama2_7b_layer", "llama2_7b_32l", "llama2_13b_128k", "llama3_8b_gqa")


def get(name: str) -> Workload:
    return WORKLOADS[name]


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields replaced (smaller test cases)."""
    return dataclasses.replace(w, **changes)


# ------------------------------------------------------------------ seeding

def _seed64(seed: int, *tags: int) -> int:
    ss = np.random.SeedSequence([int(seed) & 0xFFFFFFFF, *[int(t) & 0xFFFFFFFF for t in tags]])
    st = ss.generate_state(2, np.uint32)
    return (int(st[0]) | (int(st[1]) << 32)) & ((1 << 63) - 1)


def generator(device, seed: int, *tags: int) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(_seed64(seed, *tags))
    return g


def np_rng(seed: int, *tags: int) -> np.random.Generator:
    return np.random.default_rng(_seed64(seed, *tags))


# ------------------------------------------------------------------ shapes

def seq_lens(w: Workload, seed: int = 0) -> np.ndarray:
    if w.seq_len is not None:
        return np.full(w.num_seqs, w.seq_len, np.int32)
    lo, hi = w.seq_len_range
    return np_rng(seed, _TAG["seq_lens"]).integers(lo, hi + 1, size=w.num_seqs).astype(np.int32)


def cu_seqlens(lens: np.ndarray) -> np.ndarray:
    out = np.zeros(len(lens) + 1, np.int64)
    out[1:] = np.cumsum(lens.astype(np.int64))
    return out


def num_chunks(lens: np.ndarray, chunk_len: int) -> np.ndarray:
    return (lens.astype(np.int64) + chunk_len - 1) // chunk_len


def outlier_channels(w: Workload, seed: int = 0) -> Tuple[int, ...]:
    if w.outlier_channels is not None:
        return tuple(w.outlier_channels)
    rng = np_rng(seed, _TAG["outliers"])
    return tuple(sorted(int(c) for c in rng.choice(w.head_dim, w.num_outlier_channels,
                                                   replace=False)))


# ------------------------------------------------------------------ draws

def router_weights(w: Workload, seed: int = 0, device="cpu"):
    """W1, W2 [D, H] ~ N(0, 1/D); W3 [H, 3] ~ N(0, 1/H); b3 [3] (fixed input)."""
    D, H = w.router_dim, w.router_hidden
    W1 = torch.randn(D, H, generator=generator(device, seed, _TAG["w1"]), device=device)
    W2 = torch.randn(D, H, generator=generator(device, seed, _TAG["w2"]), device=device)
    W3 = torch.randn(H, 3, generator=generator(device, seed, _TAG["w3"]), device=device)
    W1.mul_(1.0 / np.sqrt(D))
    W2.mul_(1.0 / np.sqrt(D))
    W3.mul_(1.0 / np.sqrt(H))
    b3 = torch.tensor(w.router_bias, dtype=torch.float32, device=device)
    return W1, W2, W3, b3


def router_input(w: Workload, lens: np.ndarray, seed: int = 0, device="cpu",
                 chunk_range: Optional[Tuple[int, int]] = None) -> torch.Tensor:
    """C [rows, D] fp32 with chunk structure.

    Chunks are numbered globally (sequences back to back).  The draw is done in
    blocks of 64 chunks, so chunk_range=(c0, c1) returns exactly the rows of
    chunks c0..c1-1 of the full tensor without drawing the rest.
    """
    D, L = w.router_dim, w.chunk_len
    counts = chunk_token_counts(lens, L)
    starts = np.zeros(len(counts) + 1, np.int64)
    starts[1:] = np.cumsum(counts)
    N = len(counts)
    c0, c1 = chunk_range if chunk_range is not None else (0, N)
    a = float(np.sqrt(w.chunk_corr))
    b = float(np.sqrt(1.0 - w.chunk_corr))
    out = torch.empty(int(starts[c1] - starts[c0]), D, dtype=torch.float32, device=device)
    blk = _CHUNK_BLOCK
    for cb in range(c0 // blk, (c1 + blk - 1) // blk):
        blo, bhi = cb * blk, min((cb + 1) * blk, N)
        zc = torch.randn(blk, D, generator=generator(device, seed, _TAG["c_chunk"], cb),
                         device=device)
        zt = torch.randn(int(starts[bhi] - starts[blo]), D,
                         generator=generator(device, seed, _TAG["c_token"], cb), device=device)
        chunk_of_row = torch.as_tensor(np.repeat(np.arange(bhi - blo), counts[blo:bhi]),
                                       device=device)
        block = zc[chunk_of_row].mul_(a).add_(zt, alpha=b)
        lo, hi = max(blo, c0), min(bhi, c1)
        out[int(starts[lo] - starts[c0]):int(starts[hi] - starts[c0])] = \
            block[int(starts[lo] - starts[blo]):int(starts[hi] - starts[blo])]
    return out


_CHUNK_BLOCK = 64


def similarity_query(w: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    """u [B, D] fp32 ~ N(0, I): one query vector per sequence."""
    return torch.randn(w.num_seqs, w.router_dim, generator=generator(device, seed, _TAG["u"]),
                       device=device)


def similarity_thresholds(w: Workload) -> Tuple[float, float]:
    """(tau_hi, tau_lo) putting about target_mix of the chunks in FP16 / INT4 /
    INT2 when the cosine is close to N(0, 1/D) (independent query)."""
    from statistics import NormalDist
    f16, _, f2 = w.target_mix
    sd = 1.0 / np.sqrt(w.router_dim)
    nd = NormalDist()
    return float(nd.inv_cdf(1.0 - f16) * sd), float(nd.inv_cdf(f2) * sd)


def chunk_token_counts(lens: np.ndarray, L: int) -> np.ndarray:
    """Tokens of every chunk, sequences back to back (the tail chunk may be short)."""
    lens = np.asarray(lens, np.int64)
    n = (lens + L - 1) // L
    counts = np.full(int(n.sum()), L, np.int64)
    ends = np.cumsum(n)
    for T, e, nb in zip(lens.tolist(), ends.tolist(), n.tolist()):
        if nb > 0:
            counts[e - 1] = T - (nb - 1) * L
    return counts


def kv_layer(w: Workload, lens: np.ndarray, layer: int = 0, seed: int = 0, device="cpu"):
    """K, V [T, Hkv, d] in the workload's dtype; K carries the outlier channels
    and the token-0 sink of every sequence."""
    T = int(lens.sum())
    shape = (T, w.num_kv_heads, w.head_dim)
    s = seed + layer
    K = torch.randn(*shape, generator=generator(device, s, _TAG["k"]), device=device)
    V = torch.randn(*shape, generator=generator(device, s, _TAG["v"]), device=device)
    ch = torch.as_tensor(outlier_channels(w, seed), device=device, dtype=torch.long)
    K[:, :, ch] *= w.outlier_scale
    if w.sink_scale != 1.0:
        first = torch.as_tensor(cu_seqlens(lens)[:-1][lens > 0], device=device, dtype=torch.long)
        K[first] *= w.sink_scale
    return K.to(w.torch_dtype), V.to(w.torch_dtype)


def query(w: Workload, layer: int = 0, step: int = 0, seed: int = 0, device="cpu"):
    """q [B, Hq, d] in the workload's dtype; a fresh draw per (layer, step)."""
    q = torch.randn(w.num_seqs, w.num_q_heads, w.head_dim,
                    generator=generator(device, seed + layer, _TAG["q"], step), device=device)
    return q.to(w.torch_dtype)


def new_token_kv(w: Workload, layer: int = 0, step: int = 0, seed: int = 0, device="cpu"):
    """K, V [B, Hkv, d] of the token each sequence appends at decode step
    `step` (a fresh draw per (layer, step), the workload's dtype)."""
    shape = (w.num_seqs, w.num_kv_heads, w.head_dim)
    K = torch.randn(*shape, generator=generator(device, seed + layer, _TAG["k_new"], step),
                    device=device)
    V = torch.randn(*shape, generator=generator(device, seed + layer, _TAG["v_new"], step),
                    device=device)
    return K.to(w.torch_dtype), V.to(w.torch_dtype)


def new_token_router_input(w: Workload, step: int = 0, seed: int = 0, device="cpu"):
    """Router input rows [B, D] fp32 of the tokens appended at decode step `step`."""
    return torch.randn(w.num_seqs, w.router_dim,
                       generator=generator(device, seed, _TAG["c_new"], step), device=device)


def synthetic_chunk_map(lens: np.ndarray, chunk_len: int, mix=(0.2, 0.5, 0.3), seed: int = 0,
                        freeze_first: bool = True) -> np.ndarray:
    """A random chunk map with the given mix (an input for layout/pack/decode
    checks that must not depend on routing).  Chunk 0 is FP16 when
    freeze_first."""
    nch = num_chunks(lens, chunk_len)
    rng = np_rng(seed, _TAG["map"])
    m = rng.choice(3, size=int(nch.sum()), p=np.asarray(mix) / np.sum(mix)).astype(np.uint8)
    if freeze_first:
        off = 0
        for n in nch.tolist():
            if n > 0:
                m[off] = 0
            off += n
    return m
