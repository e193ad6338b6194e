"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare it with the CPU oracle.  The oracle only ever receives inputs from
the seeded generator (never a value produced by the CUDA path)."""
import dataclasses

import numpy as np
import torch

from chunk_adaptive_mixed_b200 import mqkv as M
from chunk_adaptive_mixed_b200 import workloads as W
from oracle import oracle as O

# decode attention tolerance (rel-L2 and max-abs against fp64)
REL_L2 = 1e-3
MAX_ABS = 4e-3
# router scores: tokens whose fp64 top-2 gap is below this may flip
NEAR_TIE = 1e-3
# Score error allowed against the fp64 oracle.  A token's argmax can change
# only if some score moves by half its top-2 gap or more, so any error below
# NEAR_TIE / 2 keeps every choice outside the near-tie band exact.  The
# router's three bf16 passes (~2^-16 relative per product, fp32 tensor-core
# accumulation) measure up to ~8e-5 at D = 5120; 4e-4 keeps a margin under
# NEAR_TIE / 2.
SCORE_TOL = 4e-4


def dev():
    return torch.device("cuda:0")


@dataclasses.dataclass
class Case:
    lens: np.ndarray
    Hq: int
    Hkv: int
    d: int
    L: int
    dtype: str = "f16"

    @property
    def B(self):
        return len(self.lens)

    @property
    def T(self):
        return int(np.sum(self.lens))

    @property
    def N(self):
        return int(((self.lens.astype(np.int64) + self.L - 1) // self.L).sum())

    @property
    def torch_dtype(self):
        return torch.float16 if self.dtype == "f16" else torch.float32

    def shape(self):
        return M.shape(self.B, self.Hq, self.Hkv, self.d, self.L)

    def cu(self):
        return torch.as_tensor(W.cu_seqlens(self.lens), device=dev())


def random_kv(case, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    K = torch.randn(case.T, case.Hkv, case.d, generator=g) * 1.5
    V = torch.randn(case.T, case.Hkv, case.d, generator=g)
    q = torch.randn(case.B, case.Hq, case.d, generator=g)
    if case.d > 40:
        K[:, :, 3] *= 8.0
    return K.to(case.torch_dtype), V.to(case.torch_dtype), q.to(case.torch_dtype)


# ------------------------------------------------------------- CUDA path

def gpu_route(case, C, W1, W2, W3, b3, freeze=True):
    shp = case.shape()
    te = torch.empty(max(case.T, 16), dtype=torch.uint8, device=dev())
    ce = torch.empty(max(case.N, 16), dtype=torch.uint8, device=dev())
    logits = torch.empty(max(case.T, 1), 3, dtype=torch.float32, device=dev())
    ws = torch.empty(M.mq_route_workspace_bytes(shp, case.lens, C.shape[1], W1.shape[1]),
                     dtype=torch.uint8, device=dev())
    M.mq_route_chunks(shp, case.lens, case.cu(), C, W1, W2, W3, b3, te, ce, ws, logits,
                      routing_freeze=freeze)
    torch.cuda.synchronize()
    assert M.mq_device_status() == 0
    return (te[:case.T].cpu().numpy(), ce[:case.N].cpu().numpy(),
            logits[:case.T].cpu().numpy())


def gpu_layout(case, chunk_expert):
    shp = case.shape()
    ce = torch.as_tensor(np.concatenate([chunk_expert, np.zeros(16, np.uint8)]), device=dev())
    layout = torch.zeros(M.mq_layout_bytes(shp, case.lens), dtype=torch.uint8, device=dev())
    M.mq_build_layout(shp, case.lens, case.cu(), ce, layout)
    return layout


def gpu_pack(case, layout, K, V):
    pb = M.mq_packed_bytes(layout)
    packed = torch.zeros(max(pb, 16), dtype=torch.uint8, device=dev())
    M.mq_pack_kv(case.shape(), case.lens, layout, K, V, packed)
    torch.cuda.synchronize()
    assert M.mq_device_status() == 0
    return packed, pb


def gpu_decode(case, layout, packed, q, scale=0.0):
    out = torch.full((case.B, case.Hq, case.d), float("nan"), dtype=torch.float32, device=dev())
    ws = torch.empty(M.mq_decode_workspace_bytes(case.shape(), case.lens), dtype=torch.uint8,
                     device=dev())
    M.mq_decode_attn(case.shape(), case.lens, layout, packed, q, out, ws, softmax_scale=scale)
    torch.cuda.synchronize()
    assert M.mq_device_status() == 0
    return out.cpu().numpy()


# ------------------------------------------------------------- comparisons

SCHEDULE_HEADER = [(28, 32), (48, 60)]
SCHEDULE_SEQ = [(128, 152)]


def strip_schedule(blob, B):
    b = np.array(blob, np.uint8, copy=True)
    for lo, hi in SCHEDULE_HEADER:
        b[lo:hi] = 0
    for s in range(B):
        base = O.HEADER_BYTES + s * O.SEQ_BYTES
        for lo, hi in SCHEDULE_SEQ:
            b[base + lo:base + hi] = 0
    return b


def check_schedule(blob, case):
    """The decode split is implementation-defined: check it is a valid cover."""
    h, seqs, _, _ = O.parse_layout(blob, case.B)
    it = h["item_tokens"]
    assert all(x >= 32 and x % 32 == 0 for x in it)
    nxt = 0
    for s in seqs:
        for e in range(3):
            n = s["seg_tokens"][e]
            c = s["item_count"][e]
            assert s["item_begin"][e] == nxt
            assert c * it[e] >= n and (c == 0 or (c - 1) * it[e] < n)
            nxt += c
    assert h["total_items"] == nxt


def check_layout(case, gpu_blob, chunk_expert):
    ob, pb = O.build_layout(case.Hkv, case.d, case.L, case.lens, chunk_expert)
    assert np.array_equal(strip_schedule(gpu_blob, case.B), ob), "layout table differs"
    check_schedule(gpu_blob, case)
    return ob, pb


def check_attention(gpu, ref, what=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(gpu)), what
    diff = gpu - ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30)
    mx = float(np.abs(diff).max()) if diff.size else 0.0
    assert rel <= REL_L2 and mx <= MAX_ABS, f"{what}: rel-L2 {rel:.3e}, max-abs {mx:.3e}"
    return rel, mx


def check_route(lens, L, te_gpu, ce_gpu, logits_gpu, z32, z64, freeze=True):
    """Maps must agree except where the oracle's own fp64 scores are within
    NEAR_TIE of a tie.  Returns (near-tie tokens, exempt chunks)."""
    te_o = O.token_argmax(z32)
    gap = O.top2_gap(z64)
    near = gap < NEAR_TIE
    scale = np.maximum(1.0, np.abs(z64))
    assert np.all(np.abs(logits_gpu - z64) <= SCORE_TOL * scale), \
        f"router scores differ: max {np.abs(logits_gpu - z64).max():.3e}"
    bad = (te_gpu != te_o) & ~near
    assert not bad.any(), f"{bad.sum()} token choices differ away from ties"
    ce_o = O.vote(lens, L, te_o, routing_freeze=freeze)
    # chunk exemption: the vote margin is within the number of near-tie tokens
    exempt = 0
    row = 0
    ci = 0
    for T in np.asarray(lens).tolist():
        nb = (T + L - 1) // L
        for c in range(nb):
            t0, t1 = row + c * L, row + min((c + 1) * L, T)
            cnt = np.bincount(te_o[t0:t1], minlength=3)
            top2 = np.sort(cnt)[-2:]
            margin = top2[1] - top2[0]
            if ce_gpu[ci + c] != ce_o[ci + c]:
                assert margin <= near[t0:t1].sum() and not (freeze and c == 0), \
                    f"chunk {ci + c} differs with margin {margin}"
                exempt += 1
        row += T
        ci += nb
    return int(near.sum()), exempt


def packed_row(packed_np, seqs, inv, L, Hkv, d, b, t, kv, g, e, chunk_offset):
    """Bytes of one encoded row (codes, scales) at the place the header's
    format puts them (addresses from the oracle's layout)."""
    s = seqs[b]
    c = t // L
    p = int(inv[chunk_offset + c])
    row = (p - s["seg_chunk_begin"][e]) * L + (t - c * L)
    base = s["seg_base"][e] + (kv * Hkv + g) * s["region_bytes"][e]
    rb = d * (16, 4, 2)[e] // 8
    codes = packed_np[base + row * rb: base + (row + 1) * rb]
    if e == 0:
        return codes, None
    so = base + s["scale_offset"][e] + row * (d // 32) * 4
    return codes, packed_np[so: so + (d // 32) * 4]


def oracle_row(x_row, e):
    """The oracle's encoding of one row (numpy float32 of d values)."""
    d = len(x_row)
    if e == 0:
        return O.f32_to_f16(x_row).view(np.uint8), None
    bits = (4, 2)[e - 1]
    codes = []
    scales = []
    for k in range(d // 32):
        c, _, _, sh, mh = O.quantize_group(x_row[32 * k:32 * k + 32], bits)
        codes.append(O.pack_codes(c, bits))
        scales.append(np.array([sh, mh], np.uint16).view(np.uint8))
    return np.concatenate(codes), np.concatenate(scales)
