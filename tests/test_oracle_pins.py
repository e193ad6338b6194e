"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks the oracle against a closed form, an identity of the
mathematics, exact rational arithmetic, a special case with a known answer, an
invariant of the method, or bytes derived by hand from the public header's
format.  None of these runs the CUDA library.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LN3 = math.log(3.0)


# ----------------------------------------------------------------- router

def test_router_zero_w1_gives_bias_exactly():
    # W1 = 0 -> SiLU(0) = 0 -> gated hidden is 0 -> scores are exactly b3
    rng = np.random.default_rng(1)
    T, D, H = 7, 12, 8
    C = rng.standard_normal((T, D)).astype(np.float32)
    W1 = np.zeros((D, H), np.float32)
    W2 = rng.standard_normal((D, H)).astype(np.float32)
    W3 = rng.standard_normal((H, 3)).astype(np.float32)
    b3 = np.array([0.25, -1.5, 0.75], np.float32)
    z32, z64 = O.router_logits(C, W1, W2, W3, b3)
    assert np.array_equal(z32, np.tile(b3, (T, 1)))
    assert np.array_equal(z64, np.tile(b3.astype(np.float64), (T, 1)))
    assert np.all(O.token_argmax(z32) == 2)


def test_router_sigmoid_special_points_and_orientation():
    # sigma(ln 3) = 3/4 and sigma(-ln 3) = 1/4, so with (C W1) = (ln3, 0, -ln3)
    # and (C W2) = (4/ln3, 5, 8/ln3) the gated hidden is exactly (3, 0, -2).
    # D=2, H=3 and a non-symmetric W3 make a transposed operand or swapped
    # branches give a different answer.
    a = np.float32(LN3)
    C = np.array([[1.0, 0.5]], np.float32)
    W1 = np.array([[a, 0.0, -a], [0.0, 0.0, 0.0]], np.float32)
    W2 = np.array([[4.0 / a, 5.0, 8.0 / a], [0.0, 0.0, 0.0]], np.float32)
    W3 = np.array([[1.0, 0.0, 2.0], [7.0, 7.0, 7.0], [0.0, 1.0, 1.0]], np.float32)
    b3 = np.array([0.5, 0.0, -1.0], np.float32)
    _, z64 = O.router_logits(C, W1, W2, W3, b3)
    # g = (3, 0, -2):  z = g W3 + b3 = (3, -2, 4) + b3
    expect = np.array([3.0 + 0.5, -2.0, 4.0 - 1.0])
    assert np.allclose(z64[0], expect, rtol=0, atol=2e-6), z64


def test_router_odd_part_is_bilinear():
    # SiLU(x) - SiLU(-x) = x, hence z(C) + z(-C) - 2 b3 = ((C W1) * (C W2)) W3:
    # with small integers the right side is exact.
    rng = np.random.default_rng(2)
    T, D, H = 5, 6, 4
    C = rng.integers(-3, 4, (T, D)).astype(np.float32)
    W1 = rng.integers(-2, 3, (D, H)).astype(np.float32)
    W2 = rng.integers(-2, 3, (D, H)).astype(np.float32)
    W3 = rng.integers(-2, 3, (H, 3)).astype(np.float32)
    b3 = np.array([1.0, -2.0, 0.5], np.float32)
    _, zp = O.router_logits(C, W1, W2, W3, b3)
    _, zn = O.router_logits(-C, W1, W2, W3, b3)
    Ci, W1i, W2i, W3i = (x.astype(np.int64) for x in (C, W1, W2, W3))
    rhs = ((Ci @ W1i) * (Ci @ W2i)) @ W3i
    lhs = zp + zn - 2.0 * b3.astype(np.float64)
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-9), (lhs, rhs)


def test_router_large_argument_limit():
    # SiLU(x) -> x for large x (error x*exp(-x) < 1e-15 at x = 40)
    C = np.array([[1.0]], np.float32)
    W1 = np.array([[40.0, 41.0]], np.float32)
    W2 = np.array([[2.0, -1.0]], np.float32)
    W3 = np.array([[1.0, 0.0, 0.0], [0.0, 1.0, 1.0]], np.float32)
    _, z64 = O.router_logits(C, W1, W2, W3, None)
    assert np.allclose(z64[0], [80.0, -41.0, -41.0], atol=1e-12)


def test_token_argmax_ties_go_to_more_bits():
    z = np.array([[0.5, 0.5, 0.5], [0.0, 1.0, 1.0], [0.0, 0.5, 1.0], [2.0, 1.0, 2.0],
                  [-1.0, -1.0, -2.0]], np.float32)
    assert O.token_argmax(z).tolist() == [0, 1, 2, 0, 0]


def test_top2_gap():
    z = np.array([[0.5, 0.5, 0.1], [3.0, 1.0, 2.0]], np.float64)
    assert np.allclose(O.top2_gap(z), [0.0, 1.0])


def test_vote_majority_ties_tail_and_freeze():
    L = 64
    # seq 0: 2 full chunks + tail of 3 tokens; seq 1: 1 chunk of 40 tokens
    lens = np.array([131, 40], np.int32)
    te = np.zeros(171, np.uint8)
    te[0:64] = 2                       # chunk 0: all INT2 (frozen to FP16)
    te[64:96] = 1
    te[96:128] = 2                     # chunk 1: 32/32 INT4/INT2 tie -> INT4
    te[128:131] = [0, 1, 2]            # tail: three-way tie -> FP16
    te[131:171] = 2
    te[131:140] = 1                    # seq 1 chunk 0: 9 INT4, 31 INT2 -> INT2
    assert O.vote(lens, L, te, routing_freeze=True).tolist() == [0, 1, 0, 0]
    assert O.vote(lens, L, te, routing_freeze=False).tolist() == [2, 1, 0, 2]


def test_route_end_to_end_special_case():
    # W1 = 0 -> scores = b3 -> every token and chunk takes argmax(b3);
    # routing freezing still pins chunk 0 of every sequence to FP16
    lens = np.array([300, 64, 1], np.int32)
    T, D, H = int(lens.sum()), 8, 64
    rng = np.random.default_rng(3)
    C = rng.standard_normal((T, D)).astype(np.float32)
    W1 = np.zeros((D, H), np.float32)
    W2 = rng.standard_normal((D, H)).astype(np.float32)
    W3 = rng.standard_normal((H, 3)).astype(np.float32)
    ce, te, _, _ = O.route(lens, 64, C, W1, W2, W3, np.array([0, 0, 1], np.float32), True)
    assert te.tolist() == [2] * T
    assert ce.tolist() == [0, 2, 2, 2, 2, 0, 0]
    ce, _, _, _ = O.route(lens, 64, C, W1, W2, W3, np.array([1, 1, 1], np.float32), False)
    assert ce.tolist() == [0] * 7


# ----------------------------------------------------------------- layout

def _random_case(seed, B=5, L=64):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, 9 * L, B).astype(np.int32)
    lens[0] = 4 * L  # one exact multiple
    n = int(((lens + L - 1) // L).sum())
    ce = rng.integers(0, 3, n).astype(np.uint8)
    return lens, ce


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
@pytest.mark.parametrize("d", [64, 128])
def test_layout_invariants(seed, d):
    L, Hkv = 64, 3
    lens, ce = _random_case(seed, L=L)
    blob, pb = O.build_layout(Hkv, d, L, lens, ce)
    h, seqs, perm, inv = O.parse_layout(blob, len(lens))
    assert h["magic"] == 0x4C4B514D and h["version"] == 1
    assert h["total_chunks"] == len(ce) and h["total_tokens"] == int(lens.sum())
    assert h["packed_bytes"] == pb == O.packed_bytes(Hkv, d, L, lens, ce)
    base = 0
    for b, s in enumerate(seqs):
        Tb = int(lens[b])
        nb = (Tb + L - 1) // L
        off = s["chunk_offset"]
        assert s["num_tokens"] == Tb and s["num_chunks"] == nb
        assert s["token_offset"] == int(lens[:b].sum())
        m = ce[off:off + nb]
        p = perm[off:off + nb]
        iv = inv[off:off + nb]
        assert sorted(p.tolist()) == list(range(nb))            # permutation
        assert all(iv[p[i]] == i for i in range(nb))            # inverse
        assert sum(s["seg_chunks"]) == nb and sum(s["seg_tokens"]) == Tb
        pos = 0
        for e in range(3):
            assert s["seg_chunk_begin"][e] == pos
            seg = p[pos:pos + s["seg_chunks"][e]]
            assert all(m[c] == e for c in seg)                  # one precision
            assert list(seg) == sorted(seg)                     # stable order
            toks = sum(min(L, Tb - c * L) for c in seg)
            assert s["seg_tokens"][e] == toks
            if nb and (nb - 1) in seg:
                assert seg[-1] == nb - 1                        # tail chunk last
            pos += s["seg_chunks"][e]
            # region geometry, from the header's formulas
            n = s["seg_tokens"][e]
            a128 = lambda x: (x + 127) // 128 * 128  # noqa: E731
            if e == 0:
                assert s["scale_offset"][0] == 0
                assert s["region_bytes"][0] == a128(n * 2 * d)
            else:
                bits = (4, 2)[e - 1]
                assert s["scale_offset"][e] == a128(n * d * bits // 8)
                assert s["region_bytes"][e] == a128(n * d * bits // 8) + a128(n * (d // 32) * 4)
            assert s["seg_base"][e] == base
            base += 2 * Hkv * s["region_bytes"][e]
            assert s["seg_base"][e] % 128 == 0
    assert base == pb


def test_fp16_cache_size_matches_the_papers_claim():
    # MoQAE notes, 研究背景: a 128k context of Llama2-13B needs a KV cache of
    # about 100 GB.  40 layers x (K+V) x 40 heads x 128 dims x 131072 tokens x
    # 2 bytes = 107,374,182,400 bytes = 100 GiB.
    lens = np.array([131072], np.int32)
    ce = np.zeros(512, np.uint8)
    per_layer = O.packed_bytes(40, 128, 256, lens, ce)
    assert per_layer * 40 == 40 * 2 * 40 * 128 * 131072 * 2 == 100 * 2 ** 30


@pytest.mark.parametrize("e,eff_bits", [(0, 16), (1, 5), (2, 3)])
def test_effective_bits_closed_form(e, eff_bits):
    # INT4 stores 4 bits + one 32-bit (scale, min) per 32 values = 5 bits/value;
    # INT2 -> 3 bits; FP16 -> 16 bits (aligned case: no padding)
    lens = np.array([4096], np.int32)
    ce = np.full(32, e, np.uint8)
    pb = O.packed_bytes(8, 128, 128, lens, ce)
    assert pb * 8 == eff_bits * 2 * 8 * 128 * 4096


def test_avgbit_of_a_map():
    # AvgBit (MoQAE notes, main table) = sum of chunk bits / number of chunks
    ce = np.array([0, 1, 1, 2, 1, 2, 2, 1], np.uint8)
    bits = np.array(O.EXPERT_BITS)[ce]
    assert bits.sum() / len(ce) == (16 + 4 * 4 + 2 * 3) / 8


# -------------------------------------------------------------- quantiser

def _rn32(fr: Fraction) -> np.float32:
    """Round a rational to the nearest float32 (ties to even), exactly."""
    f = np.float32(float(fr))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    best = min(cands, key=lambda c: (abs(Fraction(float(c)) - fr),
                                     int(np.array(c).view(np.uint32)) & 1))
    return best


def _groups(rng, n, kind):
    out = []
    for _ in range(n):
        if kind == "f16":
            x = rng.standard_normal(32).astype(np.float16).astype(np.float32)
        elif kind == "f32":
            x = (rng.standard_normal(32) * rng.uniform(0.01, 50)).astype(np.float32)
        else:  # coarse values: many exact midpoints / ties
            x = (rng.integers(-8, 9, 32) / 4).astype(np.float32)
        out.append(x)
    return out


@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("kind", ["f16", "f32", "coarse"])
def test_quantiser_is_nearest_level_exactly(bits, kind):
    rng = np.random.default_rng(10 + bits)
    levels = (1 << bits) - 1
    near_half = 0
    total = 0
    for x in _groups(rng, 150, kind):
        codes, s, mn, sh, mh = O.quantize_group(x, bits)
        lo, hi = Fraction(float(x.min())), Fraction(float(x.max()))
        assert float(mn) == float(x.min())
        if lo == hi:
            assert s == 1.0 and np.all(codes == 0)
            continue
        # s is the fp32 rounding of RN32(max - min) / levels, computed exactly
        span32 = np.float32(x.max()) - np.float32(x.min())   # IEEE fp32 subtract
        assert s == _rn32(Fraction(float(span32)) / levels)
        sf = Fraction(float(s))
        for j in range(32):
            r = (Fraction(float(x[j])) - lo) / sf           # exact ratio
            k = math.floor(r)
            frac = r - k
            if frac > Fraction(1, 2):
                ideal = k + 1
            elif frac < Fraction(1, 2):
                ideal = k
            else:
                ideal = k if k % 2 == 0 else k + 1
            ideal = min(max(ideal, 0), levels)
            total += 1
            if codes[j] != ideal:
                # only where fp32 rounding of (x - mn) / s can cross a .5
                assert abs(frac - Fraction(1, 2)) <= Fraction(1, 2 ** 19), (x[j], r)
                near_half += 1
    # realistic inputs hit that window rarely; the coarse grid is built to hit it
    if kind != "coarse":
        assert near_half <= total // 100


@pytest.mark.parametrize("bits", [4, 2])
def test_quantiser_extremes_and_error_bounds(bits):
    rng = np.random.default_rng(20 + bits)
    levels = (1 << bits) - 1
    for x in _groups(rng, 200, "f16") + _groups(rng, 100, "f32"):
        codes, s, mn, sh, mh = O.quantize_group(x, bits)
        if x.max() == x.min():
            continue
        assert codes[int(np.argmin(x))] == 0
        assert codes[int(np.argmax(x))] == levels
        xd = x.astype(np.float64)
        s64, mn64 = float(s), float(mn)
        err = np.abs(xd - (codes * s64 + mn64))
        assert np.all(err <= s64 / 2 * (1 + 2 ** -18) + 1e-30)
        # with the stored fp16 parameters
        sh64 = float(np.array(sh, np.uint16).view(np.float16))
        mh64 = float(np.array(mh, np.uint16).view(np.float16))
        bound = sh64 / 2 + levels * abs(s64 - sh64) + abs(mn64 - mh64)
        err_h = np.abs(xd - (codes * sh64 + mh64))
        assert np.all(err_h <= bound * (1 + 2 ** -18) + 1e-30)


def test_constant_group():
    x = np.full(32, -1.25, np.float32)
    for bits in (4, 2):
        codes, s, mn, sh, mh = O.quantize_group(x, bits)
        assert s == 1.0 and mn == -1.25 and np.all(codes == 0)
        assert sh == 0x3C00 and mh == np.array(-1.25, np.float16).view(np.uint16)


def _golden_bits():
    rows = {}
    with open(os.path.join(GOLDEN, "pack_bit_order.txt")) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            k, v = line.split(":")
            rows[k.strip()] = bytes(int(t, 16) for t in v.split())
    return rows


def test_bit_order_matches_hand_derived_bytes():
    g = _golden_bits()
    assert bytes(O.pack_codes(np.arange(32) % 16, 4)) == g["int4 ramp"]
    assert bytes(O.pack_codes(np.arange(32) % 4, 2)) == g["int2 ramp"]
    one = np.zeros(32, np.uint8)
    one[9] = 15
    assert bytes(O.pack_codes(one, 4)) == g["int4 one"]
    one = np.zeros(32, np.uint8)
    one[17] = 3
    assert bytes(O.pack_codes(one, 2)) == g["int2 one"]


@pytest.mark.parametrize("bits", [4, 2])
def test_pack_unpack_round_trip(bits):
    rng = np.random.default_rng(bits)
    for _ in range(50):
        c = rng.integers(0, 1 << bits, 32).astype(np.uint8)
        assert np.array_equal(O.unpack_codes(O.pack_codes(c, bits), bits), c)


def test_fp16_rounding_is_round_to_nearest_even():
    # hand-picked cases with known IEEE answers
    cases = {1.0 + 2.0 ** -11: 1.0,                 # tie -> even (1.0)
             1.0 + 3 * 2.0 ** -11: 1.0 + 2.0 ** -9,  # tie -> even (up)
             65504.0: 65504.0, 65519.0: 65504.0,     # largest finite
             2.0 ** -25: 0.0,                        # tie between 0 and 2^-24 -> 0
             3 * 2.0 ** -26: 2.0 ** -24,             # above the tie -> 2^-24
             -1.0 - 2.0 ** -11: -1.0}
    xs = np.array(list(cases), np.float32)
    got = O.f32_to_f16(xs).astype(np.float64)
    assert got.tolist() == list(cases.values())
    assert np.isinf(O.f32_to_f16(np.array([65520.0], np.float32))[0])
    # and agrees with numpy's independent conversion on many values
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-18, 11, 200000))).astype(np.float32)
    with np.errstate(over="ignore"):  # values beyond 65520 overflow to infinity on both sides
        want = x.astype(np.float16)
    assert np.array_equal(O.f32_to_f16(x).view(np.uint16), want.view(np.uint16))


# ------------------------------------------------------------ full pack

def _unpack_region_token(packed, seqs, b, e, kv, g, Hkv, d, row):
    """Reads one token row back out of a packed buffer using the header's
    format description (independently of the oracle's C code)."""
    s = seqs[b]
    base = s["seg_base"][e] + (kv * Hkv + g) * s["region_bytes"][e]
    if e == 0:
        raw = packed[base + row * 2 * d: base + (row + 1) * 2 * d]
        return raw.view(np.float16).astype(np.float64), None, None
    bits = (4, 2)[e - 1]
    rb = d * bits // 8
    raw = packed[base + row * rb: base + (row + 1) * rb]
    codes = np.concatenate([O.unpack_codes(raw[4 * bits * k: 4 * bits * (k + 1)], bits)
                            for k in range(d // 32)])
    sc = packed[base + s["scale_offset"][e] + row * (d // 32) * 4:
                base + s["scale_offset"][e] + (row + 1) * (d // 32) * 4].view(np.float16)
    return codes, sc[0::2].astype(np.float64), sc[1::2].astype(np.float64)


@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_pack_places_every_row_where_the_header_says(dtype):
    L, Hkv, d = 64, 2, 64
    lens, ce = _random_case(7, B=3, L=L)
    rng = np.random.default_rng(8)
    T = int(lens.sum())
    K = rng.standard_normal((T, Hkv, d)).astype(dtype)
    V = rng.standard_normal((T, Hkv, d)).astype(dtype)
    packed = O.pack(Hkv, d, L, lens, ce, K, V)
    blob, pb = O.build_layout(Hkv, d, L, lens, ce)
    assert pb == len(packed)
    _, seqs, perm, inv = O.parse_layout(blob, len(lens))
    for b in range(len(lens)):
        s = seqs[b]
        for t in range(0, int(lens[b]), 5):
            c = t // L
            e = int(ce[s["chunk_offset"] + c])
            p = int(inv[s["chunk_offset"] + c])
            row = (p - s["seg_chunk_begin"][e]) * L + (t - c * L)
            for kv, src in ((0, K), (1, V)):
                for g in range(Hkv):
                    x = src[s["token_offset"] + t, g].astype(np.float32)
                    codes, sc, mn = _unpack_region_token(packed, seqs, b, e, kv, g, Hkv, d, row)
                    if e == 0:
                        # FP16 rows: fp16 input is copied, fp32 input rounded
                        assert np.array_equal(codes, x.astype(np.float16).astype(np.float64))
                        continue
                    bits = (4, 2)[e - 1]
                    for k in range(d // 32):
                        qc, _, _, sh, mh = O.quantize_group(x[32 * k:32 * k + 32], bits)
                        assert np.array_equal(codes[32 * k:32 * k + 32], qc)
                        assert sc[k] == np.array(sh, np.uint16).view(np.float16)
                        assert mn[k] == np.array(mh, np.uint16).view(np.float16)


# -------------------------------------------------------------- attention

def _attn_case(B, Hq, Hkv, d, lens, dtype, seed):
    rng = np.random.default_rng(seed)
    T = int(np.sum(lens))
    K = rng.standard_normal((T, Hkv, d)).astype(dtype)
    V = rng.standard_normal((T, Hkv, d)).astype(dtype)
    q = rng.standard_normal((B, Hq, d)).astype(dtype)
    return K, V, q


def test_dense_attention_two_token_closed_form():
    # scores differ by exactly ln 3 -> weights 1/4, 3/4
    d = 64
    K = np.zeros((2, 1, d), np.float32)
    V = np.zeros((2, 1, d), np.float32)
    K[1, 0, 0] = np.float32(LN3)
    V[0, 0, :] = 4.0
    V[1, 0, :] = -8.0
    q = np.zeros((1, 1, d), np.float32)
    q[0, 0, 0] = 1.0
    o = O.dense_attention(1, 1, d, [2], K, V, q, scale=1.0)
    assert np.allclose(o[0, 0], 0.25 * 4.0 + 0.75 * -8.0, atol=1e-6)
    # default scale is 1/sqrt(d): same answer once q is scaled by sqrt(d)
    o2 = O.dense_attention(1, 1, d, [2], K, V, q * np.float32(8.0), scale=0.0)
    assert np.allclose(o2, o, atol=1e-6)


@pytest.mark.parametrize("e", [0, 1, 2])
def test_decode_single_token_returns_its_value(e):
    L, d, Hkv, Hq = 64, 64, 2, 4
    lens = np.array([1], np.int32)
    K, V, q = _attn_case(1, Hq, Hkv, d, lens, np.float16, 30)
    ce = np.array([e], np.uint8)
    packed = O.pack(Hkv, d, L, lens, ce, K, V)
    o = O.decode(Hq, Hkv, d, L, lens, ce, packed, q)
    blob, _ = O.build_layout(Hkv, d, L, lens, ce)
    _, seqs, _, _ = O.parse_layout(blob, 1)
    for h in range(Hq):
        codes, sc, mn = _unpack_region_token(packed, seqs, 0, e, 1, h // 2, Hkv, d, 0)
        v = codes if e == 0 else codes * np.repeat(sc, 32) + np.repeat(mn, 32)
        assert np.array_equal(o[0, h], v)


def _dequant_values(packed, seqs, inv, ce, L, Hkv, d, Tb, kv, g):
    out = []
    for t in range(Tb):
        c = t // L
        e = int(ce[c])
        row = (int(inv[c]) - seqs[0]["seg_chunk_begin"][e]) * L + t - c * L
        codes, sc, mn = _unpack_region_token(packed, seqs, 0, e, kv, g, Hkv, d, row)
        out.append(codes if e == 0 else codes * np.repeat(sc, 32) + np.repeat(mn, 32))
    return np.asarray(out)


@pytest.mark.parametrize("case", ["equal_keys_one_precision", "zero_query_mixed"])
def test_decode_uniform_weights_give_mean_value(case):
    # equal dequantised keys (same rows, same precision) or a zero query make
    # every softmax weight equal: the output is the mean of the values
    L, d, Hkv, Hq = 64, 128, 1, 2
    lens = np.array([200], np.int32)
    K, V, q = _attn_case(1, Hq, Hkv, d, lens, np.float16, 31)
    if case == "equal_keys_one_precision":
        K[:] = K[0]
        ce = np.array([2, 2, 2, 2], np.uint8)
    else:
        ce = np.array([0, 1, 2, 1], np.uint8)
        q[:] = 0
    packed = O.pack(Hkv, d, L, lens, ce, K, V)
    o = O.decode(Hq, Hkv, d, L, lens, ce, packed, q)
    blob, _ = O.build_layout(Hkv, d, L, lens, ce)
    _, seqs, _, inv = O.parse_layout(blob, 1)
    mean = _dequant_values(packed, seqs, inv, ce, L, Hkv, d, 200, 1, 0).mean(axis=0)
    assert np.allclose(o[0, 0], mean, rtol=0, atol=1e-12)
    assert np.allclose(o[0, 1], mean, rtol=0, atol=1e-12)


def test_decode_all_fp16_equals_dense_attention():
    L, d, Hkv, Hq = 32, 64, 2, 4
    lens = np.array([70, 0, 33], np.int32)
    K, V, q = _attn_case(3, Hq, Hkv, d, lens, np.float16, 33)
    n = int(((lens + L - 1) // L).sum())
    ce = np.zeros(n, np.uint8)
    packed = O.pack(Hkv, d, L, lens, ce, K, V)
    o = O.decode(Hq, Hkv, d, L, lens, ce, packed, q)
    dense = O.dense_attention(Hq, Hkv, d, lens, K, V, q)
    assert np.allclose(o, dense, rtol=0, atol=1e-13)
    assert np.all(o[1] == 0.0)  # empty sequence -> zeros


def test_decode_is_invariant_to_chunk_order():
    L, d, Hkv, Hq = 64, 64, 1, 2
    lens = np.array([6 * 64], np.int32)
    K, V, q = _attn_case(1, Hq, Hkv, d, lens, np.float16, 34)
    ce = np.array([0, 2, 1, 1, 2, 0], np.uint8)
    o = O.decode(Hq, Hkv, d, L, lens, ce, O.pack(Hkv, d, L, lens, ce, K, V), q)
    order = [3, 0, 5, 1, 4, 2]
    Kp = np.concatenate([K[c * L:(c + 1) * L] for c in order])
    Vp = np.concatenate([V[c * L:(c + 1) * L] for c in order])
    cp = ce[order]
    op = O.decode(Hq, Hkv, d, L, lens, cp, O.pack(Hkv, d, L, lens, cp, Kp, Vp), q)
    assert np.allclose(o, op, rtol=0, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv():
    L, d, Hkv, Hq = 64, 64, 2, 8
    lens = np.array([150, 64], np.int32)
    K, V, q = _attn_case(2, Hq, Hkv, d, lens, np.float16, 35)
    ce = np.array([0, 1, 2, 2, 0], np.uint8)
    o = O.decode(Hq, Hkv, d, L, lens, ce, O.pack(Hkv, d, L, lens, ce, K, V), q)
    Kr = np.repeat(K, Hq // Hkv, axis=1)
    Vr = np.repeat(V, Hq // Hkv, axis=1)
    om = O.decode(Hq, Hq, d, L, lens, ce, O.pack(Hq, d, L, lens, ce, Kr, Vr), q)
    assert np.array_equal(o, om)


def test_decode_pairs_agrees_with_decode():
    L, d, Hkv, Hq = 64, 128, 2, 4
    lens = np.array([130, 257], np.int32)
    K, V, q = _attn_case(2, Hq, Hkv, d, lens, np.float16, 36)
    ce = np.array([0, 1, 2, 0, 2, 1, 1, 2], np.uint8)
    o = O.decode(Hq, Hkv, d, L, lens, ce, O.pack(Hkv, d, L, lens, ce, K, V), q)
    pairs = np.array([[b, h] for b in range(2) for h in range(Hq)], np.int32)
    op = O.decode_pairs(Hq, Hkv, d, L, lens, ce, K, V, q, pairs)
    assert np.array_equal(op.reshape(2, Hq, d), o)


# ------------------------------------------------------ similarity search

def test_similarity_route_closed_forms():
    # chunk rows built as exact multiples of u: cos = +1, -1, 0 (orthogonal)
    D, L = 8, 32
    u = np.zeros((1, D), np.float32)
    u[0, :4] = [1.0, 2.0, -1.0, 0.5]
    ortho = np.zeros(D, np.float32)
    ortho[4:] = [3.0, -1.0, 2.0, 1.0]                  # disjoint support: orthogonal to u
    rows = []
    for c, v in enumerate([u[0] * 2.0, -u[0], ortho, u[0] + 0.0 * ortho]):
        rows.append(np.tile(v, (L, 1)))
    C = np.concatenate(rows).astype(np.float32)
    lens = np.array([4 * L], np.int32)
    ce, sim = O.similarity_route(lens, L, C, u, tau_hi=0.9, tau_lo=-0.5, routing_freeze=False)
    assert np.allclose(sim, [1.0, -1.0, 0.0, 1.0], atol=1e-12)
    assert ce.tolist() == [0, 2, 1, 0]
    ce, _ = O.similarity_route(lens, L, C, u, tau_hi=0.9, tau_lo=-0.5, routing_freeze=True)
    assert ce.tolist() == [0, 2, 1, 0]
    # the similarity uses the chunk MEAN: varying rows whose mean is u give 1
    noise = np.random.default_rng(0).standard_normal((L, D)).astype(np.float32)
    noise -= noise.mean(axis=0, keepdims=True)
    C2 = (np.tile(u[0], (L, 1)) + noise).astype(np.float64)
    C2 -= C2.mean(axis=0) - u[0]                      # exact mean = u (up to fp32)
    _, sim2 = O.similarity_route(np.array([L], np.int32), L, C2.astype(np.float32), u, 0.5, 0.0,
                                 routing_freeze=False)
    assert abs(sim2[0] - 1.0) < 1e-6


def test_similarity_route_tail_zero_and_freeze():
    D, L = 4, 32
    u = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 0.0, 0.0, 0.0]], np.float32)
    lens = np.array([40, 5], np.int32)                # tail chunk of 8 tokens; second seq u = 0
    C = np.zeros((45, D), np.float32)
    C[32:40, 0] = -2.0                                # tail chunk anti-aligned
    C[40:45, 1] = 1.0
    ce, sim = O.similarity_route(lens, L, C, u, tau_hi=0.5, tau_lo=0.25, routing_freeze=False)
    assert sim.tolist() == [0.0, -1.0, 0.0]           # zero mean chunk 0, tail -1, u = 0
    assert ce.tolist() == [2, 2, 2]
    ce, _ = O.similarity_route(lens, L, C, u, tau_hi=0.5, tau_lo=0.25, routing_freeze=True)
    assert ce.tolist() == [0, 2, 0]


# ------------------------------------------------------ context-split records

def test_decode_partial_two_token_closed_form():
    # K rows a multiple of e0, q = 2 e0: scores scale * 2 * x_t; all FP16, exact in fp16
    d, L = 64, 32
    K = np.zeros((2, 1, d), np.float32)
    V = np.zeros((2, 1, d), np.float32)
    K[0, 0, 0], K[1, 0, 0] = 1.5, -0.75
    V[0, 0, 1], V[1, 0, 2] = 1.0, 1.0
    q = np.zeros((1, 1, d), np.float32)
    q[0, 0, 0] = 2.0
    lens = np.array([2], np.int32)
    ce = np.zeros(1, np.uint8)
    ref = O.pack(1, d, L, lens, ce, K, V)
    o, ml = O.decode_partial(1, 1, d, L, lens, ce, ref, q)
    s = np.array([3.0, -1.5]) / np.sqrt(d)
    assert abs(ml[0, 0, 0] - s[0]) < 1e-15
    assert abs(ml[0, 0, 1] - (1.0 + np.exp(s[1] - s[0]))) < 1e-15
    p = np.exp(s - s.max()) / np.exp(s - s.max()).sum()
    assert np.allclose(o[0, 0, 1:3], p, atol=1e-15)


def test_decode_partial_records_merge_to_the_whole_sequence():
    # a sequence cut at a chunk boundary: the two shards' records, merged with
    # the split-softmax rule, give the attention over the whole sequence
    rng = np.random.default_rng(5)
    d, L, Hkv, Hq = 64, 32, 2, 4
    T, cut = 5 * L - 7, 2 * L
    K = (rng.standard_normal((T, Hkv, d)) * 1.3).astype(np.float32)
    V = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    q = rng.standard_normal((1, Hq, d)).astype(np.float32)
    cmap = np.array([0, 2, 1, 1, 2], np.uint8)
    full = np.array([T], np.int32)
    ref = O.pack(Hkv, d, L, full, cmap, K, V)
    o_full, ml_full = O.decode_partial(Hq, Hkv, d, L, full, cmap, ref, q)
    recs = []
    for lo, hi, m in [(0, cut, cmap[:2]), (cut, T, cmap[2:])]:
        lens = np.array([hi - lo], np.int32)
        r = O.pack(Hkv, d, L, lens, m, K[lo:hi], V[lo:hi])
        recs.append(O.decode_partial(Hq, Hkv, d, L, lens, m, r, q))
    M = np.maximum(recs[0][1][..., 0], recs[1][1][..., 0])
    w = [ml[..., 1] * np.exp(ml[..., 0] - M) for _, ml in recs]
    merged = (w[0][..., None] * recs[0][0] + w[1][..., None] * recs[1][0]) / (w[0] + w[1])[..., None]
    assert np.allclose(merged, o_full, rtol=0, atol=1e-12)
    assert np.allclose(M, ml_full[..., 0], atol=1e-14)
    assert np.allclose(w[0] + w[1], ml_full[..., 1], rtol=1e-12)
    # an empty shard contributes nothing
    z = O.decode_partial(Hq, Hkv, d, L, np.array([0], np.int32), np.zeros(0, np.uint8),
                         np.zeros(16, np.uint8), q)
    assert np.all(z[1][..., 0] == -np.inf) and np.all(z[1][..., 1] == 0) and np.all(z[0] == 0)


# ------------------------------------------------------------ threads

def test_oracle_results_do_not_depend_on_its_thread_count():
    # every parallel loop of the oracle runs over independent outputs (tokens,
    # chunks, (sequence, head) pairs), each summed serially in a fixed order,
    # so the host's core count cannot change a stored or compared value
    rng = np.random.default_rng(7)
    lens = np.array([300, 0, 77, 513], np.int32)
    Hq, Hkv, d, L, D, H = 8, 2, 64, 32, 48, 16
    T = int(lens.sum())
    C = rng.standard_normal((T, D)).astype(np.float32)
    W1 = (rng.standard_normal((D, H)) / np.sqrt(D)).astype(np.float32)
    W2 = (rng.standard_normal((D, H)) / np.sqrt(D)).astype(np.float32)
    W3 = (rng.standard_normal((H, 3)) / np.sqrt(H)).astype(np.float32)
    K = rng.standard_normal((T, Hkv, d)).astype(np.float16)
    V = rng.standard_normal((T, Hkv, d)).astype(np.float16)
    q = rng.standard_normal((len(lens), Hq, d)).astype(np.float16)

    def run():
        z32, _ = O.router_logits(C, W1, W2, W3)
        cmap = O.route(lens, L, C, W1, W2, W3)[0]
        packed = O.pack(Hkv, d, L, lens, cmap, K, V)
        return z32, cmap, packed, O.decode(Hq, Hkv, d, L, lens, cmap, packed, q)

    prev = O.num_threads()
    try:
        O.set_num_threads(1)
        one = run()
        O.set_num_threads(max(4, prev))
        many = run()
    finally:
        O.set_num_threads(prev)
    for a, b in zip(one, many):
        assert np.array_equal(np.asarray(a).view(np.uint8), np.asarray(b).view(np.uint8))
