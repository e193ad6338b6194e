"""Decode-time cache growth (mq_grow_*) against the CPU oracle.

The grown cache must hold exactly what a fresh build would hold for the grown
sequences with the same chunk map — the open tail in FP16, every sealed
chunk at the expert it was sealed with — so the oracle side is the plain
oracle layout / pack / decode of that state (chunks quantised from the tail
use the tail's fp16 values).  Compared: decode outputs at several steps, and
at the end the layout counts, perm / inv and every packed row (bit-exact).
"""
import numpy as np
import pytest
import torch

from chunk_adaptive_mixed_b200 import mqkv as M
from chunk_adaptive_mixed_b200 import workloads as W
from oracle import oracle as O

from .gpu_helpers import Case, check_attention, dev, packed_row

pytestmark = pytest.mark.gpu

NO_SEAL = 255


class Mirror:
    """Host copy of the grown state, for the oracle."""

    def __init__(self, case, cmap, K, V, layers):
        self.case = case
        L = case.L
        self.lens = case.lens.astype(np.int64).copy()
        self.full0 = self.lens // L                      # chunks complete at prefill
        starts = np.concatenate([[0], np.cumsum((case.lens + L - 1) // L)])
        self.maps = []
        for b in range(case.B):
            m = list(cmap[starts[b]:starts[b + 1]])
            if case.lens[b] % L:
                m[-1] = 0                                # the open tail is FP16
            self.maps.append(m)
        cu = W.cu_seqlens(case.lens)
        self.K = [[K[l][cu[b]:cu[b + 1]].clone() for b in range(case.B)] for l in range(layers)]
        self.V = [[V[l][cu[b]:cu[b + 1]].clone() for b in range(case.B)] for l in range(layers)]

    def append(self, layer, Kn, Vn):
        for b in range(self.case.B):
            self.K[layer][b] = torch.cat([self.K[layer][b], Kn[b:b + 1]])
            self.V[layer][b] = torch.cat([self.V[layer][b], Vn[b:b + 1]])

    def add_token(self):
        L = self.case.L
        for b in range(self.case.B):
            if self.lens[b] % L == 0:
                self.maps[b].append(0)                   # a new open tail
            self.lens[b] += 1

    def seal(self, b, e):
        self.maps[b][-1] = e

    def state(self, layer):
        """(lens, flat map, K, V) of the current state; tail tokens in fp16."""
        L = self.case.L
        Ks, Vs = [], []
        for b in range(self.case.B):
            k, v = self.K[layer][b].clone(), self.V[layer][b].clone()
            t0 = int(self.full0[b]) * L                  # tokens after this were in the tail
            k[t0:] = k[t0:].half().to(k.dtype)
            v[t0:] = v[t0:].half().to(v.dtype)
            Ks.append(k)
            Vs.append(v)
        flat = np.array([e for m in self.maps for e in m], np.uint8)
        return (self.lens.astype(np.int32), flat, torch.cat(Ks).numpy(), torch.cat(Vs).numpy())


def _oracle_decode(case, mirror, layer, q):
    lens, flat, K, V = mirror.state(layer)
    ref = O.pack(case.Hkv, case.d, case.L, lens, flat, K, V)
    return O.decode(case.Hq, case.Hkv, case.d, case.L, lens, flat, ref, q)


def _grow_fields(blob, B):
    h = int(np.asarray(blob[60:64]).view(np.int32)[0])
    st = []
    for b in range(B):
        base = O.HEADER_BYTES + b * O.SEQ_BYTES
        st.append(np.asarray(blob[base + 152:base + 160]).view(np.int32).tolist())
    return h, st


def _run_growth(case, grow, steps, layers=2, seed=0, check_every=17):
    dtype = case.torch_dtype
    shp = case.shape()
    g = torch.Generator().manual_seed(seed)
    K = [torch.randn(case.T, case.Hkv, case.d, generator=g).to(dtype) for _ in range(layers)]
    V = [torch.randn(case.T, case.Hkv, case.d, generator=g).to(dtype) for _ in range(layers)]
    cmap = W.synthetic_chunk_map(case.lens, case.L, mix=(0.3, 0.4, 0.3), seed=seed)
    mirror = Mirror(case, cmap, K, V, layers)
    rng = np.random.default_rng(seed)

    lay_b, pk_b, ws_b = M.mq_grow_sizes(shp, case.lens, grow)
    cap_lens = case.lens + grow
    layout = torch.zeros(lay_b, dtype=torch.uint8, device=dev())
    ce = torch.as_tensor(np.concatenate([cmap, np.zeros(16, np.uint8)]), device=dev())
    M.mq_grow_build_layout(shp, case.lens, grow, case.cu(), ce, layout)
    packed = [torch.zeros(pk_b, dtype=torch.uint8, device=dev()) for _ in range(layers)]
    for l in range(layers):
        M.mq_grow_pack_kv(shp, case.lens, grow, layout, K[l].to(dev()), V[l].to(dev()), packed[l])
    ws = torch.empty(ws_b, dtype=torch.uint8, device=dev())
    out = torch.empty(case.B, case.Hq, case.d, dtype=torch.float32, device=dev())
    sealed_dev = torch.full((max(case.B, 16),), NO_SEAL, dtype=torch.uint8, device=dev())
    pending = False
    checked = 0
    for s in range(steps):
        M.mq_grow_commit(shp, layout, sealed_dev if pending else None, True)
        mirror.add_token()
        for l in range(layers):
            Kn = torch.randn(case.B, case.Hkv, case.d, generator=g).to(dtype)
            Vn = torch.randn(case.B, case.Hkv, case.d, generator=g).to(dtype)
            q = torch.randn(case.B, case.Hq, case.d, generator=g).to(dtype)
            M.mq_grow_append_kv(shp, layout, Kn.to(dev()), Vn.to(dev()), packed[l])
            mirror.append(l, Kn, Vn)
            if s % check_every == 0 or s == steps - 1:
                M.mq_decode_attn(shp, cap_lens, layout, packed[l], q.to(dev()), out, ws)
                torch.cuda.synchronize()
                assert M.mq_device_status() == 0, f"step {s}"
                want = _oracle_decode(case, mirror, l, q.numpy())
                check_attention(out.cpu().numpy(), want, f"step {s} layer {l}")
                checked += 1
        # seal every tail that is now full
        sealed = np.full(max(case.B, 16), NO_SEAL, np.uint8)
        for b in range(case.B):
            if mirror.lens[b] % case.L == 0:
                c = int(mirror.lens[b]) // case.L - 1
                e = 0 if c == 0 else int(rng.integers(0, 3))   # chunk 0: routing freezing
                sealed[b] = e
                mirror.seal(b, e)
        pending = bool((sealed[:case.B] != NO_SEAL).any())
        if pending:
            sealed_dev.copy_(torch.as_tensor(sealed))
            for l in range(layers):
                M.mq_grow_seal(shp, layout, sealed_dev, packed[l])
    # apply the last seals without adding a token, then compare everything
    M.mq_grow_commit(shp, layout, sealed_dev if pending else None, False)
    torch.cuda.synchronize()
    assert M.mq_device_status() == 0
    return mirror, layout, packed, checked


def _check_final_state(case, mirror, layout, packed, layers):
    blob = layout.cpu().numpy()
    h, seqs, perm, inv = O.parse_layout(blob, case.B)
    lens, flat, _, _ = mirror.state(0)
    ob, pb = O.build_layout(case.Hkv, case.d, case.L, lens, flat)
    oh, oseqs, operm, oinv = O.parse_layout(ob, case.B)
    assert h["total_tokens"] == int(lens.sum())
    for b in range(case.B):
        for key in ("num_tokens", "num_chunks", "seg_chunks", "seg_chunk_begin", "seg_tokens"):
            assert seqs[b][key] == oseqs[b][key], (b, key, seqs[b][key], oseqs[b][key])
        n = seqs[b]["num_chunks"]
        c0, o0 = seqs[b]["chunk_offset"], oseqs[b]["chunk_offset"]
        assert np.array_equal(perm[c0:c0 + n], operm[o0:o0 + n]), b
        assert np.array_equal(inv[c0:c0 + n], oinv[o0:o0 + n]), b
    grow_chunks, st = _grow_fields(blob, case.B)
    assert grow_chunks > 0
    for l in range(layers):
        _, _, K, V = mirror.state(l)
        ref = O.pack(case.Hkv, case.d, case.L, lens, flat, K, V)
        got = packed[l].cpu().numpy()
        for b in range(case.B):
            mb = mirror.maps[b]
            for t in range(int(lens[b])):
                c = t // case.L
                e = mb[c]
                for kv in range(2):
                    for gh in range(case.Hkv):
                        a = packed_row(got, seqs, inv, case.L, case.Hkv, case.d, b, t, kv, gh, e,
                                       seqs[b]["chunk_offset"])
                        w = packed_row(ref, oseqs, oinv, case.L, case.Hkv, case.d, b, t, kv, gh, e,
                                       oseqs[b]["chunk_offset"])
                        assert np.array_equal(a[0], w[0]), (l, b, t, kv, gh, "codes")
                        if e:
                            assert np.array_equal(a[1], w[1]), (l, b, t, kv, gh, "scales")


@pytest.mark.parametrize("d,L,dtype", [(128, 64, "f16"), (64, 32, "f32")])
def test_growth_matches_a_fresh_build(d, L, dtype):
    # a partial tail, a sequence ending on a chunk boundary, an empty sequence
    lens = np.array([300, 4 * L, 0], np.int32)
    case = Case(lens, 4, 2, d, L, dtype)
    steps = 3 * L + 5
    mirror, layout, packed, checked = _run_growth(case, grow=steps, steps=steps)
    assert checked >= 2 * (steps // 17)
    assert all(len(m) == (int(n) + L - 1) // L for m, n in zip(mirror.maps, mirror.lens))
    _check_final_state(case, mirror, layout, packed, layers=2)


def test_growth_capacity_overflow_is_reported_without_faults():
    L = 32
    case = Case(np.array([40], np.int32), 2, 2, 64, L, "f16")
    shp = case.shape()
    lay_b, pk_b, _ = M.mq_grow_sizes(shp, case.lens, 1)
    layout = torch.zeros(lay_b, dtype=torch.uint8, device=dev())
    ce = torch.zeros(16, dtype=torch.uint8, device=dev())
    M.mq_grow_build_layout(shp, case.lens, 1, case.cu(), ce, layout)
    packed = torch.zeros(pk_b, dtype=torch.uint8, device=dev())
    K = torch.randn(40, 2, 64).half().to(dev())
    M.mq_grow_pack_kv(shp, case.lens, 1, layout, K, K, packed)
    torch.cuda.synchronize()
    assert M.mq_device_status() == 0
    Kn = torch.randn(1, 2, 64).half().to(dev())
    seen = None
    for s in range(4 * L):          # never sealed: the FP16 rows run out
        M.mq_grow_commit(shp, layout, None, True)
        M.mq_grow_append_kv(shp, layout, Kn, Kn, packed)
        torch.cuda.synchronize()
        st = M.mq_device_status()
        if st:
            seen = (s, st)
            break
    assert seen is not None and seen[1] == M.MQ_DEV_CAPACITY, seen
    _, grow_state = _grow_fields(layout.cpu().numpy(), 1)
    assert grow_state[0][1] & M.MQ_GROW_FULL


def test_commit_on_a_fixed_layout_is_rejected_on_the_device():
    case = Case(np.array([100], np.int32), 2, 2, 64, 32, "f16")
    shp = case.shape()
    layout = torch.zeros(M.mq_layout_bytes(shp, case.lens), dtype=torch.uint8, device=dev())
    ce = torch.zeros(16, dtype=torch.uint8, device=dev())
    M.mq_build_layout(shp, case.lens, case.cu(), ce, layout)
    before = layout.clone()
    M.mq_grow_commit(shp, layout, None, True)
    torch.cuda.synchronize()
    assert M.mq_device_status() == M.MQ_DEV_BAD_LAYOUT
    assert torch.equal(before, layout)
