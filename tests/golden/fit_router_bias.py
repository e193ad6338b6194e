"""Chooses each workload's router bias b3 with the CPU oracle.

b3 is an input of the router (a fixed per-expert offset after W3).  The
workloads give only a target chunk mix (e.g. ~15/60/25 % FP16/INT4/INT2), so
this script draws a sample of chunks of each workload, evaluates the oracle's
router scores once without bias, and searches b3 = (0, b1, b2) on a grid so
that the oracle's per-token argmax and per-chunk vote give the mix closest to
the target (sum of absolute differences, frozen chunks left out).  The values
it prints are copied into chunk_adaptive_mixed_b200/workloads.py; the CPU test
test_workload_mix re-checks them with the oracle.

Usage: python tests/golden/fit_router_bias.py [workload ...]
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from chunk_adaptive_mixed_b200 import workloads as W  # noqa: E402
from oracle import oracle as O  # noqa: E402

SAMPLE_CHUNKS = {"tiny": 16, "llama2_7b_layer": 32, "llama2_7b_32l": 256,
                 "llama2_13b_128k": 128, "llama3_8b_gqa": 256}


def sample(w, seed=0):
    lens = W.seq_lens(w, seed)
    n = int(W.num_chunks(lens, w.chunk_len).sum())
    c1 = min(n, SAMPLE_CHUNKS[w.name])
    C = W.router_input(w, lens, seed, "cpu", chunk_range=(0, c1)).numpy()
    counts = W.chunk_token_counts(lens, w.chunk_len)[:c1].astype(np.int32)
    # first chunk of every sequence inside the sample is frozen to FP16 by the
    # method; leave those out of the statistic
    starts = np.cumsum(np.concatenate([[0], W.num_chunks(lens, w.chunk_len)]))
    frozen = np.zeros(c1, bool)
    frozen[starts[:-1][starts[:-1] < c1]] = True
    W1, W2, W3, _ = W.router_weights(w, seed, "cpu")
    z32, _ = O.router_logits(C, W1.numpy(), W2.numpy(), W3.numpy(), None)
    return z32, counts, frozen


def mix_for(z32, counts, frozen, bias):
    z = (z32 + np.asarray(bias, np.float32)).astype(np.float32)
    te = O.token_argmax(z)
    ce = O.vote(counts, int(counts.max()), te, routing_freeze=False)
    ce = ce[~frozen]
    return np.bincount(ce, minlength=3) / max(len(ce), 1)


def fit(w, seed=0):
    z32, counts, frozen = sample(w, seed)
    target = np.asarray(w.target_mix)
    best = (9.0, (0.0, 0.0, 0.0))
    for step, span, center in ((0.05, 1.5, (0.0, 0.0)), (0.01, 0.1, None), (0.002, 0.02, None)):
        c = center if center is not None else best[1][1:]
        grid = np.arange(-span, span + 1e-9, step)
        for b1 in c[0] + grid:
            for b2 in c[1] + grid:
                m = mix_for(z32, counts, frozen, (0.0, b1, b2))
                err = float(np.abs(m - target).sum())
                if err < best[0] - 1e-12:
                    best = (err, (0.0, round(float(b1), 4), round(float(b2), 4)))
    m = mix_for(z32, counts, frozen, best[1])
    return best[1], m, best[0]


if __name__ == "__main__":
    names = sys.argv[1:] or list(W.WORKLOAD_ORDER)
    for name in names:
        w = W.get(name)
        b, m, err = fit(w)
        print(f"{name}: router_bias={b}  mix={np.round(m, 3).tolist()}  "
              f"target={list(w.target_mix)}  l1={err:.3f}", flush=True)
