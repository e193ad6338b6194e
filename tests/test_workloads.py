"""Checks of the seeded input generator (CPU only).

The generator holds no method arithmetic; these tests check its recipe
(shapes, distributions, determinism) and, with the CPU oracle, that each
workload's fixed router bias gives a chunk mix near the stated target.
"""
import numpy as np
import pytest
import torch

from chunk_adaptive_mixed_b200 import workloads as W
from oracle import oracle as O


def test_shapes_and_lengths():
    w = W.get("llama3_8b_gqa")
    lens = W.seq_lens(w)
    assert lens.shape == (64,) and lens.min() >= 2048 and lens.max() <= 16384
    assert np.array_equal(lens, W.seq_lens(w))            # deterministic
    assert W.cu_seqlens(lens)[-1] == lens.sum()
    w = W.get("tiny")
    K, V = W.kv_layer(w, W.seq_lens(w))
    assert K.shape == (1024, 4, 64) and K.dtype == torch.float32


def test_outliers_and_sink():
    w = W.get("llama2_7b_layer")
    lens = W.seq_lens(w)
    K, V = W.kv_layer(w, lens)
    assert K.dtype == torch.float16
    ch = list(W.outlier_channels(w))
    Kf = K[1:].float()
    assert 8.5 < Kf[:, :, ch].std().item() < 11.5
    other = [c for c in range(128) if c not in ch]
    assert 0.9 < Kf[:, :, other].std().item() < 1.1
    assert 4.0 < (K[0].float()[:, other].std() / Kf[:, :, other].std()).item() < 6.0
    assert 0.9 < V.float().std().item() < 1.1


def test_router_input_is_chunk_structured_and_sampleable():
    w = W.get("tiny")
    lens = W.seq_lens(w)
    C = W.router_input(w, lens)
    assert C.shape == (1024, 256)
    assert abs(C.std().item() - 1.0) < 0.05
    # rows inside a chunk correlate (rho ~ 0.9), rows of different chunks do not
    a, b, c = C[0], C[1], C[64]
    assert torch.dot(a, b).item() / 256 > 0.7
    assert abs(torch.dot(a, c).item() / 256) < 0.3
    assert torch.equal(W.router_input(w, lens, chunk_range=(5, 9)), C[5 * 64:9 * 64])


def test_layers_and_steps_differ():
    w = W.get("tiny")
    lens = W.seq_lens(w)
    K0, _ = W.kv_layer(w, lens, layer=0)
    K1, _ = W.kv_layer(w, lens, layer=1)
    assert not torch.equal(K0, K1)
    assert not torch.equal(W.query(w, step=0), W.query(w, step=1))


@pytest.mark.parametrize("name,chunks", [("tiny", 16), ("llama2_7b_layer", 32),
                                         ("llama3_8b_gqa", 64)])
def test_workload_mix_near_target(name, chunks):
    w = W.get(name)
    lens = W.seq_lens(w)
    C = W.router_input(w, lens, chunk_range=(0, chunks)).numpy()
    counts = W.chunk_token_counts(lens, w.chunk_len)[:chunks].astype(np.int32)
    W1, W2, W3, b3 = W.router_weights(w)
    z32, _ = O.router_logits(C, W1.numpy(), W2.numpy(), W3.numpy(), b3.numpy())
    ce = O.vote(counts, int(counts.max()), O.token_argmax(z32), routing_freeze=False)
    mix = np.bincount(ce, minlength=3) / len(ce)
    assert np.abs(mix - np.asarray(w.target_mix)).max() < 0.12, mix


@pytest.mark.parametrize("name", ["tiny", "llama2_13b_128k"])
def test_similarity_thresholds_give_the_target_mix(name):
    # many sequences of a few chunks each, so the mix is measured over ~256 chunks
    w = W.scaled(W.get(name), num_seqs=256, seq_len=2 * W.get(name).chunk_len,
                 seq_len_range=None, router_dim=256)
    lens = W.seq_lens(w)
    C = W.router_input(w, lens).numpy()
    u = W.similarity_query(w).numpy()
    assert u.shape == (256, 256)
    tau_hi, tau_lo = W.similarity_thresholds(w)
    assert tau_hi > tau_lo
    ce, sim = O.similarity_route(lens, w.chunk_len, C, u, tau_hi, tau_lo, routing_freeze=False)
    assert abs(sim.std() * np.sqrt(w.router_dim) - 1.0) < 0.15   # cos ~ N(0, 1/D)
    mix = np.bincount(ce, minlength=3) / len(ce)
    assert np.abs(mix - np.asarray(w.target_mix)).max() < 0.08, mix
