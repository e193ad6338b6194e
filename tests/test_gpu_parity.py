"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Small and ragged cases are compared element by element: router scores and
maps (near-ties exempt), the whole layout table (bit-exact; the decode split
checked for validity), every packed byte (bit-exact), every attention output
(rel-L2 <= 1e-3, max-abs <= 4e-3 against fp64).  The five workloads at full
size are in test_gpu_full_size.py.
"""
import zlib

import numpy as np
import pytest
import torch

from chunk_adaptive_mixed_b200 import mqkv as M
from chunk_adaptive_mixed_b200 import workloads as W
from oracle import oracle as O

from .gpu_helpers import (Case, check_attention, check_layout, check_route, dev, gpu_decode,
                          gpu_layout, gpu_pack, gpu_route, random_kv)

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_like_f32": Case(np.array([1024], np.int32), 4, 4, 64, 64, "f32"),
    "ragged_gqa4": Case(np.array([0, 1, 127, 128, 129, 1000, 3000], np.int32), 32, 8, 128, 128),
    "short_chunks": Case(np.array([2048, 33], np.int32), 16, 16, 128, 32),
    "gqa8_d64_L256": Case(np.array([5000, 257], np.int32), 8, 1, 64, 256),
    "gqa2_f32": Case(np.array([700, 64, 1], np.int32), 4, 2, 128, 64, "f32"),
    "gqa2_f16": Case(np.array([700, 64, 1, 0], np.int32), 4, 2, 128, 64, "f16"),
    "gqa8_d128": Case(np.array([2000, 33], np.int32), 16, 2, 128, 128, "f16"),
    "gqa4_d64": Case(np.array([1500, 17, 96], np.int32), 8, 2, 64, 32, "f16"),
    # fp32 queries with 4 and 8 query heads per kv-head: the CUDA-core kernel
    # with 8- and 4-dim lane slices (code words of 1 to 4 bytes)
    "gqa4_f32_d64": Case(np.array([900, 31, 64], np.int32), 8, 2, 64, 32, "f32"),
    "gqa8_f32_d128": Case(np.array([700, 129], np.int32), 16, 2, 128, 64, "f32"),
    # one query head per kv-head, fp16 queries, d = 128: the tensor-core
    # kernel of that case (16-token stages: tails of 1, 15, 16, 17 tokens)
    "mha_f16_d128": Case(np.array([0, 1, 15, 16, 17, 127, 129, 1000, 3000], np.int32), 4, 4, 128,
                         32, "f16"),
    # four query heads per kv-head, fp16 queries, d = 128: the grouped-query
    # tensor-core kernel (tails of 1 to 33 tokens around its 16/32-token stages)
    "gqa4_f16_tails": Case(np.array([1, 15, 16, 17, 31, 32, 33, 700, 0], np.int32), 8, 2, 128, 32,
                           "f16"),
}

MAPS = {"mixed": (0.2, 0.5, 0.3), "fp16": (1, 0, 0), "int4": (0, 1, 0), "int2": (0, 0, 1)}


def _map(case, mix, seed=0):
    return W.synthetic_chunk_map(case.lens, case.L, mix=mix, seed=seed, freeze_first=False)


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("mapname", list(MAPS))
def test_layout_pack_decode_parity(name, mapname):
    case = CASES[name]
    if mapname != "mixed" and name not in ("ragged_gqa4", "tiny_like_f32", "gqa8_d128", "gqa4_d64",
                                           "gqa4_f32_d64", "gqa8_f32_d128", "mha_f16_d128",
                                           "gqa4_f16_tails"):
        pytest.skip("single-precision maps run on two cases")
    cmap = _map(case, MAPS[mapname], seed=zlib.crc32(name.encode()) & 0xFFFF)
    K, V, q = random_kv(case, seed=len(name))
    layout = gpu_layout(case, cmap)
    blob = layout.cpu().numpy()
    _, pb = check_layout(case, blob, cmap)
    packed, gpb = gpu_pack(case, layout, K.to(dev()), V.to(dev()))
    assert gpb == pb
    ref = O.pack(case.Hkv, case.d, case.L, case.lens, cmap, K.numpy(), V.numpy())
    got = packed[:pb].cpu().numpy()
    if not np.array_equal(got, ref):
        bad = np.nonzero(got != ref)[0]
        raise AssertionError(f"{len(bad)} packed bytes differ, first at {bad[:8]}")
    out = gpu_decode(case, layout, packed, q.to(dev()))
    want = O.decode(case.Hq, case.Hkv, case.d, case.L, case.lens, cmap, ref, q.numpy())
    check_attention(out, want, f"{name}/{mapname}")
    empty = case.lens == 0
    assert np.all(out[empty] == 0.0)


def test_decode_softmax_scale_argument():
    case = CASES["gqa2_f32"]
    cmap = _map(case, MAPS["mixed"])
    K, V, q = random_kv(case, seed=3)
    layout = gpu_layout(case, cmap)
    packed, _ = gpu_pack(case, layout, K.to(dev()), V.to(dev()))
    ref = O.pack(case.Hkv, case.d, case.L, case.lens, cmap, K.numpy(), V.numpy())
    for scale in (0.05, 0.3):
        out = gpu_decode(case, layout, packed, q.to(dev()), scale=scale)
        want = O.decode(case.Hq, case.Hkv, case.d, case.L, case.lens, cmap, ref, q.numpy(),
                        scale=scale)
        check_attention(out, want, f"scale {scale}")


@pytest.mark.parametrize("H", [64, 128, 256])
@pytest.mark.parametrize("D,freeze", [(36, True), (256, False), (1000, True)])
def test_route_parity(H, D, freeze):
    lens = np.array([0, 70, 300, 64, 1], np.int32)
    case = Case(lens, 4, 4, 64, 64)
    T = case.T
    g = torch.Generator().manual_seed(H * 7 + D)
    # chunk-structured inputs, as in the workloads
    C = torch.randn(T, D, generator=g)
    W1 = torch.randn(D, H, generator=g) / D ** 0.5
    W2 = torch.randn(D, H, generator=g) / D ** 0.5
    W3 = torch.randn(H, 3, generator=g) / H ** 0.5
    b3 = torch.tensor([0.0, 0.1, -0.05])
    te, ce, logits = gpu_route(case, C.to(dev()), W1.to(dev()), W2.to(dev()), W3.to(dev()),
                               b3.to(dev()), freeze)
    z32, z64 = O.router_logits(C.numpy(), W1.numpy(), W2.numpy(), W3.numpy(), b3.numpy())
    check_route(lens, case.L, te, ce, logits, z32, z64, freeze)
    if freeze:
        offs = np.concatenate([[0], np.cumsum((lens + 63) // 64)])[:-1]
        assert np.all(ce[offs[lens > 0]] == 0)


def test_route_without_bias_and_zero_w1():
    # W1 = 0 -> scores are exactly the bias (or zero): special case of the router
    lens = np.array([256], np.int32)
    case = Case(lens, 4, 4, 64, 64)
    D, H = 64, 64
    C = torch.randn(256, D)
    W1 = torch.zeros(D, H)
    W2 = torch.randn(D, H)
    W3 = torch.randn(H, 3)
    te, ce, logits = gpu_route(case, C.to(dev()), W1.to(dev()), W2.to(dev()), W3.to(dev()),
                               torch.tensor([0.0, 0.0, 0.5]).to(dev()), False)
    assert np.all(logits == np.array([0.0, 0.0, 0.5], np.float32))
    assert np.all(te == 2) and np.all(ce == 2)
    te, ce, logits = gpu_route(case, C.to(dev()), W1.to(dev()), W2.to(dev()), W3.to(dev()), None,
                               True)
    assert np.all(logits == 0.0) and np.all(te == 0) and np.all(ce == 0)


@pytest.mark.parametrize("name", ["tiny", "llama2_7b_layer"])
def test_end_to_end_small_workloads(name):
    """route -> layout -> pack -> decode on the workload's own inputs, GPU vs
    oracle.  Routing is compared as in the router tests; layout, pack and
    decode then run on the oracle's map on both sides, which equals the GPU's
    own map unless a near-tie chunk flipped, so no branch ends without a
    pack and decode comparison."""
    w = W.get(name)
    lens = W.seq_lens(w)
    case = Case(lens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.chunk_len, w.kv_dtype)
    C = W.router_input(w, lens)
    W1, W2, W3, b3 = W.router_weights(w)
    K, V = W.kv_layer(w, lens)
    q = W.query(w)
    te, ce, logits = gpu_route(case, C.to(dev()), W1.to(dev()), W2.to(dev()), W3.to(dev()),
                               b3.to(dev()))
    ce_o, te_o, z32, z64 = O.route(lens, w.chunk_len, C.numpy(), W1.numpy(), W2.numpy(),
                                   W3.numpy(), b3.numpy())
    near, exempt = check_route(lens, w.chunk_len, te, ce, logits, z32, z64)
    assert ce[0] == 0
    print(f"{name}: {case.T} tokens routed, {near} near-tie tokens, {exempt} exempt chunks")
    if not np.array_equal(ce, ce_o):
        assert exempt > 0
    # layout, pack and decode run on the oracle's map: the GPU's own map
    # unless a near-tie chunk flipped (the oracle never receives the GPU's map)
    ref = O.pack(case.Hkv, case.d, case.L, lens, ce_o, K.numpy(), V.numpy())
    want = O.decode(case.Hq, case.Hkv, case.d, case.L, lens, ce_o, ref, q.numpy())
    layout = gpu_layout(case, ce_o)
    check_layout(case, layout.cpu().numpy(), ce_o)
    packed, pb = gpu_pack(case, layout, K.to(dev()), V.to(dev()))
    assert np.array_equal(packed[:pb].cpu().numpy(), ref)
    check_attention(gpu_decode(case, layout, packed, q.to(dev())), want, name)


def test_device_checks_without_faults():
    case = CASES["short_chunks"]
    cmap = _map(case, MAPS["mixed"])
    K, V, q = random_kv(case, seed=9)
    layout = gpu_layout(case, cmap)
    pb = M.mq_packed_bytes(layout)
    small = torch.full((pb // 2,), 7, dtype=torch.uint8, device=dev())
    M.mq_pack_kv(case.shape(), case.lens, layout, K.to(dev()), V.to(dev()), small)
    torch.cuda.synchronize()
    assert M.mq_device_status() & M.MQ_DEV_PACKED_TOO_SMALL
    assert torch.all(small == 7)               # nothing written
    assert M.mq_device_status() == 0           # cleared
    bad = torch.zeros_like(layout)             # no magic
    packed = torch.zeros(pb, dtype=torch.uint8, device=dev())
    M.mq_pack_kv(case.shape(), case.lens, bad, K.to(dev()), V.to(dev()), packed)
    torch.cuda.synchronize()
    assert M.mq_device_status() & M.MQ_DEV_BAD_LAYOUT
    assert torch.all(packed == 0)


def test_stream_ordering_on_a_side_stream():
    case = CASES["ragged_gqa4"]
    cmap = _map(case, MAPS["mixed"])
    K, V, q = random_kv(case, seed=11)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        layout = gpu_layout(case, cmap)
        packed, _ = gpu_pack(case, layout, K.to(dev()), V.to(dev()))
        out = gpu_decode(case, layout, packed, q.to(dev()))
    ref = O.pack(case.Hkv, case.d, case.L, case.lens, cmap, K.numpy(), V.numpy())
    want = O.decode(case.Hq, case.Hkv, case.d, case.L, case.lens, cmap, ref, q.numpy())
    check_attention(out, want, "side stream")


def test_routing_sharing_off_gives_each_layer_its_own_map_and_layout():
    """Routing sharing off (MoQAE notes, ablation without RS): every layer has
    its own router, so its own map, layout and packed cache; each layer is
    checked against the oracle with its own map."""
    lens = np.array([700, 300], np.int32)
    case = Case(lens, 8, 4, 128, 64)
    D, H = 64, 64
    g = torch.Generator().manual_seed(77)
    C = torch.randn(case.T, D, generator=g)
    maps = []
    for layer in range(3):
        W1 = torch.randn(D, H, generator=g) / D ** 0.5
        W2 = torch.randn(D, H, generator=g) / D ** 0.5
        W3 = torch.randn(H, 3, generator=g) / H ** 0.5
        b3 = torch.tensor([0.0, 0.3, 0.1])
        te, ce, logits = gpu_route(case, C.to(dev()), W1.to(dev()), W2.to(dev()), W3.to(dev()),
                                   b3.to(dev()))
        ce_o, _, z32, z64 = O.route(lens, case.L, C.numpy(), W1.numpy(), W2.numpy(), W3.numpy(),
                                    b3.numpy())
        near, exempt = check_route(lens, case.L, te, ce, logits, z32, z64)
        print(f"layer {layer}: {near} near-tie tokens, {exempt} exempt chunks")
        if not np.array_equal(ce, ce_o):
            assert exempt > 0
        maps.append(ce_o)
        K, V, q = random_kv(case, seed=100 + layer)
        # layout, pack and decode on the oracle's map (identical to the GPU's
        # unless a near-tie chunk flipped); the oracle side uses its own map
        layout = gpu_layout(case, ce_o)
        packed, pb = gpu_pack(case, layout, K.to(dev()), V.to(dev()))
        out = gpu_decode(case, layout, packed, q.to(dev()))
        ref = O.pack(case.Hkv, case.d, case.L, lens, ce_o, K.numpy(), V.numpy())
        want = O.decode(case.Hq, case.Hkv, case.d, case.L, lens, ce_o, ref, q.numpy())
        check_layout(case, layout.cpu().numpy(), ce_o)
        assert np.array_equal(packed[:pb].cpu().numpy(), ref)
        check_attention(out, want, f"layer {layer}")
    assert any(not np.array_equal(maps[0], m) for m in maps[1:])


def _adversarial_groups(n_groups, dtype, rng):
    """Groups of 32 values chosen where an encoder goes wrong: signed zeros as
    the minimum in either order, constant groups (s = 1), fp16 subnormals,
    the largest finite fp16 values, and groups whose scaled values sit exactly
    on half-integers (round-half-even) or one ulp away from them."""
    g = np.empty((n_groups, 32), np.float32)
    for i in range(n_groups):
        kind = i % 8
        if kind == 0:                                   # zero minimum, -0 first or +0 first
            x = rng.uniform(0, 3, 32).astype(np.float32)
            j0, j1 = rng.choice(32, 2, replace=False)
            x[j0], x[j1] = (-0.0, 0.0) if i % 16 == 0 else (0.0, -0.0)
        elif kind == 1:                                 # constant group
            x = np.full(32, rng.choice([0.0, -0.0, 1.5, -7.25]), np.float32)
        elif kind == 2:                                 # fp16 subnormals and zero
            x = (rng.integers(-1023, 1024, 32) * 2.0 ** -24).astype(np.float32)
        elif kind == 3:                                 # extremes of fp16
            x = rng.choice([-65504.0, 65504.0, -1.0, 0.5, 6.1e-5], 32).astype(np.float32)
        elif kind in (4, 5):                            # half-way ties at s = 1 (INT4) / s = 1 (INT2)
            top = 15.0 if kind == 4 else 3.0
            x = (rng.integers(0, int(top), 32) + 0.5).astype(np.float32)
            x[0], x[1] = 0.0, top
        elif kind == 6:                                 # ties at a power-of-two scale
            x = ((rng.integers(0, 30, 32) + 0.5) * 0.25 - 4.0).astype(np.float32)
            x[0], x[1] = -4.0, -4.0 + 7.5
        else:                                           # plain normal values
            x = rng.standard_normal(32).astype(np.float32)
        g[i] = x
    if dtype == "f16":
        g = g.astype(np.float16).astype(np.float32)     # exactly representable inputs
    return g


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_pack_adversarial_values_bit_exact(dtype):
    case = Case(np.array([300, 64, 517], np.int32), 8, 4, 128, 32, dtype)
    rng = np.random.default_rng(42 if dtype == "f16" else 43)
    n = case.T * case.Hkv * case.d // 32
    K = _adversarial_groups(n, dtype, rng).reshape(case.T, case.Hkv, case.d)
    V = _adversarial_groups(n, dtype, rng)[::-1].copy().reshape(case.T, case.Hkv, case.d)
    Kt = torch.from_numpy(K).to(case.torch_dtype)
    Vt = torch.from_numpy(V).to(case.torch_dtype)
    for mapname, mix in MAPS.items():
        cmap = _map(case, mix, seed=7)
        layout = gpu_layout(case, cmap)
        packed, pb = gpu_pack(case, layout, Kt.to(dev()), Vt.to(dev()))
        ref = O.pack(case.Hkv, case.d, case.L, case.lens, cmap, Kt.numpy(), Vt.numpy())
        got = packed[:pb].cpu().numpy()
        if not np.array_equal(got, ref):
            bad = np.nonzero(got != ref)[0]
            raise AssertionError(f"{mapname}: {len(bad)} packed bytes differ, first at {bad[:8]}")


def _tie_groups(n_groups, bits, rng):
    """fp16 groups whose range is (2^b - 1) * m * 2^e (m odd, small): many
    values sit exactly on, or one fp16 step beside, the half-integer points
    min + (k + 1/2) s, at scales of every binade."""
    lev = 2 ** bits - 1
    g = np.empty((n_groups, 32), np.float32)
    for i in range(n_groups):
        mn = np.float16(rng.uniform(-50, 50) * 2.0 ** rng.integers(-12, 3))
        d = lev * (1 + 2 * rng.integers(0, 8)) * 2.0 ** float(rng.integers(-14, 6))
        mx = np.float16(np.float32(mn) + np.float32(d))
        s = (np.float32(mx) - np.float32(mn)) / np.float32(lev)
        pts = np.float32(mn) + (rng.integers(0, lev, 32) + np.float32(0.5)) * s
        x = pts.astype(np.float16)
        step = rng.integers(-1, 2, 32)                  # one fp16 step off, or on the point
        x = np.where(step < 0, np.nextafter(x, np.float16(-np.inf)),
                     np.where(step > 0, np.nextafter(x, np.float16(np.inf)), x))
        x = np.clip(x, mn, mx).astype(np.float32)
        x[0], x[1] = np.float32(mn), np.float32(mx)
        g[i] = x
    return g


@pytest.mark.parametrize("bits", [4, 2])
def test_pack_fp16_half_integer_quotients_bit_exact(bits):
    # the fp16 encoder derives RN(t / s) without a division; these groups put
    # the quotient on, or a rounding step beside, k + 1/2 at many scales
    case = Case(np.array([256, 96], np.int32), 4, 4, 128, 32, "f16")
    rng = np.random.default_rng(100 + bits)
    n = case.T * case.Hkv * case.d // 32
    K = _tie_groups(n, bits, rng).reshape(case.T, case.Hkv, case.d)
    V = _tie_groups(n, bits, rng).reshape(case.T, case.Hkv, case.d)
    Kt, Vt = torch.from_numpy(K).half(), torch.from_numpy(V).half()
    cmap = np.full(int(W.num_chunks(case.lens, case.L).sum()), 1 if bits == 4 else 2, np.uint8)
    layout = gpu_layout(case, cmap)
    packed, pb = gpu_pack(case, layout, Kt.to(dev()), Vt.to(dev()))
    ref = O.pack(case.Hkv, case.d, case.L, case.lens, cmap, Kt.numpy(), Vt.numpy())
    got = packed[:pb].cpu().numpy()
    bad = np.nonzero(got != ref)[0]
    assert len(bad) == 0, f"{len(bad)} packed bytes differ, first at {bad[:8]}"


@pytest.mark.parametrize("hq,hkv", [(8, 2), (4, 4)])
def test_decode_with_very_large_groups(hq, hkv):
    # groups whose range reaches ~6e4 (scale ~4e4 at INT2): products of softmax
    # weights and scales far beyond fp16 range must not overflow anywhere
    case = Case(np.array([900, 130], np.int32), hq, hkv, 128, 64, "f16")
    K, V, q = random_kv(case, seed=77)
    g = torch.Generator().manual_seed(78)
    big = torch.rand(case.T, case.Hkv, 1, generator=g) < 0.3
    V = torch.where(big, (V.float() * 20000).clamp(-65000, 65000), V.float()).half()
    K = (K.float() * 0.05).half()
    cmap = _map(case, MAPS["mixed"], seed=5)
    layout = gpu_layout(case, cmap)
    packed, pb = gpu_pack(case, layout, K.to(dev()), V.to(dev()))
    ref = O.pack(case.Hkv, case.d, case.L, case.lens, cmap, K.numpy(), V.numpy())
    assert np.array_equal(packed[:pb].cpu().numpy(), ref)
    out = gpu_decode(case, layout, packed, q.to(dev()))
    want = O.decode(case.Hq, case.Hkv, case.d, case.L, case.lens, cmap, ref, q.numpy())
    scale = np.abs(want).max()
    check_attention(out / scale, want / scale, "large groups (relative to the output range)")


@pytest.mark.parametrize("hq,hkv", [(8, 2), (4, 4)])
def test_decode_with_tiny_values(hq, hkv):
    # every group tiny (scales ~1e-6): the tensor-core path keeps its relative accuracy
    case = Case(np.array([700, 90], np.int32), hq, hkv, 128, 64, "f16")
    K, V, q = random_kv(case, seed=91)
    V = (V.float() * 2e-5).half()
    cmap = _map(case, MAPS["mixed"], seed=6)
    layout = gpu_layout(case, cmap)
    packed, pb = gpu_pack(case, layout, K.to(dev()), V.to(dev()))
    ref = O.pack(case.Hkv, case.d, case.L, case.lens, cmap, K.numpy(), V.numpy())
    out = gpu_decode(case, layout, packed, q.to(dev()))
    want = O.decode(case.Hq, case.Hkv, case.d, case.L, case.lens, cmap, ref, q.numpy())
    scale = np.abs(want).max()
    check_attention(out / scale, want / scale, "tiny values (relative to the output range)")


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2)])
def test_decode_query_extremes(hq, hkv):
    # queries at the edges of fp16: all zero, a huge element beside tiny and
    # subnormal ones, every element subnormal; the tensor-core kernels scale
    # each query by a power of two before it enters an fp16 operand
    case = Case(np.array([600, 77, 33], np.int32), hq, hkv, 128, 64, "f16")
    K, V, q = random_kv(case, seed=123)
    qf = q.float()
    qf[0, 0] = 0.0
    qf[1, 0] = torch.where(torch.arange(case.d) % 3 == 0, 3e-7, 1e-3)
    qf[1, 0, 5] = 30000.0
    qf[2, 0] = torch.linspace(-1.0, 1.0, case.d) * 2.0 ** -15
    q = qf.half()
    K = (K.float() * 0.01).half()      # keeps the 30000 query's scores finite and spread
    cmap = _map(case, MAPS["mixed"], seed=8)
    layout = gpu_layout(case, cmap)
    packed, pb = gpu_pack(case, layout, K.to(dev()), V.to(dev()))
    ref = O.pack(case.Hkv, case.d, case.L, case.lens, cmap, K.numpy(), V.numpy())
    out = gpu_decode(case, layout, packed, q.to(dev()))
    want = O.decode(case.Hq, case.Hkv, case.d, case.L, case.lens, cmap, ref, q.numpy())
    check_attention(out, want, "query extremes")


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2)])
def test_many_short_sequences(hq, hkv):
    # more sequences than one block of the work-order scan (256), many of
    # them empty or shorter than a chunk: the prefix table over several
    # blocks, sequences without items in a segment, and heads with one item
    rng = np.random.default_rng(17 + hq)
    lens = rng.integers(0, 90, size=600).astype(np.int32)
    lens[::7] = 0
    lens[5] = 1
    case = Case(lens, hq, hkv, 128, 32, "f16")
    K, V, q = random_kv(case, seed=51 + hq)
    cmap = _map(case, MAPS["mixed"], seed=3)
    layout = gpu_layout(case, cmap)
    check_layout(case, layout.cpu().numpy(), cmap)
    packed, pb = gpu_pack(case, layout, K.to(dev()), V.to(dev()))
    ref = O.pack(case.Hkv, case.d, case.L, case.lens, cmap, K.numpy(), V.numpy())
    assert np.array_equal(packed[:pb].cpu().numpy(), ref)
    out = gpu_decode(case, layout, packed, q.to(dev()))
    want = O.decode(case.Hq, case.Hkv, case.d, case.L, case.lens, cmap, ref, q.numpy())
    nz = lens > 0
    check_attention(out[nz], want[nz], "many short sequences")
    assert np.all(out[~nz] == 0.0)  # an empty sequence attends to nothing


@pytest.mark.parametrize("name", ["mha_f16_d128", "gqa4_f16_tails", "gqa8_d128", "gqa2_f32",
                                  "mha_long", "gqa4_long"])
def test_decode_is_deterministic(name):
    # every work item starts from a fresh state and the merge takes the
    # records in a fixed order, so repeated calls agree bit for bit however
    # the warps' claims interleave (fresh, uninitialised workspaces; other
    # work on the device between the calls)
    long_cases = {
        # one long sequence, few heads: many items per head, merged in slices
        "mha_long": Case(np.array([40000], np.int32), 8, 8, 128, 256, "f16"),
        "gqa4_long": Case(np.array([40000, 3000], np.int32), 16, 4, 128, 128, "f16"),
    }
    case = long_cases.get(name) or CASES[name]
    cmap = _map(case, MAPS["mixed"], seed=11)
    K, V, q = random_kv(case, seed=5)
    layout = gpu_layout(case, cmap)
    packed, pb = gpu_pack(case, layout, K.to(dev()), V.to(dev()))
    qd = q.to(dev())
    outs = []
    for i in range(3):
        noise = torch.empty(64 << 20, dtype=torch.uint8, device=dev()).fill_(i)
        outs.append(gpu_decode(case, layout, packed, qd))
        del noise
    for o in outs[1:]:
        assert np.array_equal(o.view(np.uint32), outs[0].view(np.uint32))
    if name in long_cases:
        ref = O.pack(case.Hkv, case.d, case.L, case.lens, cmap, K.numpy(), V.numpy())
        assert np.array_equal(packed[:pb].cpu().numpy(), ref)
        want = O.decode(case.Hq, case.Hkv, case.d, case.L, case.lens, cmap, ref, q.numpy())
        check_attention(outs[0], want, name)
