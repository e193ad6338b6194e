"""ctypes wrapper around the CPU oracle (mqkv_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the test suite, by the package's smoke
check and by the benchmark's CPU-baseline leg; never by the library's data path.
Every array argument is a numpy array; results come back as numpy arrays.
fp16 data travels as numpy float16 (IEEE binary16 bit patterns).
"""
import ctypes

import numpy as np

from . import build_oracle

_LIB = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_vp = ctypes.c_void_p

EXPERT_BITS = (16, 4, 2)


def lib():
    global _LIB
    if _LIB is None:
        path = build_oracle.build()
        L = ctypes.CDLL(path)
        L.mqo_num_threads.restype = ctypes.c_int
        L.mqo_set_num_threads.argtypes = [ctypes.c_int]
        L.mqo_router_logits.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _f32p, _f32p,
                                        _f32p, _f32p, _f32p, _f32p, _f64p]
        L.mqo_token_argmax.argtypes = [ctypes.c_int64, _f32p, _u8p]
        L.mqo_top2_gap.argtypes = [ctypes.c_int64, _f64p, _f64p]
        L.mqo_num_chunks.argtypes = [ctypes.c_int, _i32p, ctypes.c_int]
        L.mqo_num_chunks.restype = ctypes.c_int64
        L.mqo_vote.argtypes = [ctypes.c_int, _i32p, ctypes.c_int, _u8p, ctypes.c_int, _u8p]
        L.mqo_route.argtypes = [ctypes.c_int, _i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                _f32p, _f32p, _f32p, _f32p, _f32p, ctypes.c_int, _u8p, _u8p,
                                _f32p, _f64p]
        L.mqo_layout_bytes.argtypes = [ctypes.c_int, _i32p, ctypes.c_int]
        L.mqo_layout_bytes.restype = ctypes.c_size_t
        L.mqo_build_layout.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       _i32p, _u8p, _u8p, ctypes.c_size_t]
        L.mqo_build_layout.restype = ctypes.c_uint64
        L.mqo_packed_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       _i32p, _u8p]
        L.mqo_packed_bytes.restype = ctypes.c_uint64
        L.mqo_quantize_group.argtypes = [_f32p, ctypes.c_int, _u8p, _f32p, _f32p, _u16p, _u16p]
        L.mqo_pack_codes.argtypes = [_u8p, ctypes.c_int, _u8p]
        L.mqo_unpack_codes.argtypes = [_u8p, ctypes.c_int, _u8p]
        L.mqo_pack.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p, _u8p,
                               _vp, _vp, ctypes.c_int, _u8p, ctypes.c_uint64]
        L.mqo_pack.restype = ctypes.c_int
        L.mqo_decode.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_int, _i32p, _u8p, _u8p, _vp, ctypes.c_int,
                                 ctypes.c_double, _f64p]
        L.mqo_decode_pairs.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, _i32p, _u8p, _vp, _vp, ctypes.c_int, _vp,
                                       ctypes.c_int, ctypes.c_double, _i32p, ctypes.c_int, _f64p]
        L.mqo_dense_attention.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          _i32p, _vp, _vp, ctypes.c_int, _vp, ctypes.c_int,
                                          ctypes.c_double, _f64p]
        L.mqo_decode_partial.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, _i32p, _u8p, _u8p, _vp, ctypes.c_int,
                                         ctypes.c_double, _f64p, _f64p]
        L.mqo_similarity_route.argtypes = [ctypes.c_int, _i32p, ctypes.c_int, ctypes.c_int, _f32p,
                                           _f32p, ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                           _u8p, _f64p]
        L.mqo_f32_to_f16.argtypes = [_f32p, _u16p, ctypes.c_int64]
        L.mqo_f16_to_f32.argtypes = [_u16p, _f32p, ctypes.c_int64]
        _LIB = L
    return _LIB


def _p(a, t):
    return a.ctypes.data_as(t)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _dtype_code(a):
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.float16:
        return 1
    raise TypeError(f"expected float32 or float16, got {a.dtype}")


def num_threads():
    return lib().mqo_num_threads()


def set_num_threads(n):
    lib().mqo_set_num_threads(int(n))


def num_chunks(seq_lens, L):
    sl = _c(seq_lens, np.int32)
    return int(lib().mqo_num_chunks(len(sl), _p(sl, _i32p), int(L)))


def router_logits(C, W1, W2, W3, b3=None):
    """fp32-rounded and fp64 router scores [T, 3]."""
    C = _c(C, np.float32)
    W1, W2, W3 = _c(W1, np.float32), _c(W2, np.float32), _c(W3, np.float32)
    T, D = C.shape
    H = W1.shape[1]
    assert W1.shape == (D, H) and W2.shape == (D, H) and W3.shape == (H, 3)
    z32 = np.empty((T, 3), np.float32)
    z64 = np.empty((T, 3), np.float64)
    b3c = _c(b3, np.float32) if b3 is not None else None
    bp = _p(b3c, _f32p) if b3c is not None else None
    lib().mqo_router_logits(T, D, H, _p(C, _f32p), _p(W1, _f32p), _p(W2, _f32p), _p(W3, _f32p),
                            bp, _p(z32, _f32p), _p(z64, _f64p))
    return z32, z64


def token_argmax(z32):
    z32 = _c(z32, np.float32)
    out = np.empty(z32.shape[0], np.uint8)
    lib().mqo_token_argmax(z32.shape[0], _p(z32, _f32p), _p(out, _u8p))
    return out


def top2_gap(z64):
    z64 = _c(z64, np.float64)
    out = np.empty(z64.shape[0], np.float64)
    lib().mqo_top2_gap(z64.shape[0], _p(z64, _f64p), _p(out, _f64p))
    return out


def vote(seq_lens, L, token_expert, routing_freeze=True):
    sl = _c(seq_lens, np.int32)
    te = _c(token_expert, np.uint8)
    out = np.empty(num_chunks(sl, L), np.uint8)
    lib().mqo_vote(len(sl), _p(sl, _i32p), int(L), _p(te, _u8p), int(bool(routing_freeze)),
                   _p(out, _u8p))
    return out


def route(seq_lens, L, C, W1, W2, W3, b3=None, routing_freeze=True):
    """Returns (chunk_expert, token_expert, logits32, logits64)."""
    sl = _c(seq_lens, np.int32)
    C = _c(C, np.float32)
    W1, W2, W3 = _c(W1, np.float32), _c(W2, np.float32), _c(W3, np.float32)
    D = C.shape[1]
    H = W1.shape[1]
    T = int(sl.sum())
    assert C.shape[0] == T
    te = np.empty(T, np.uint8)
    ce = np.empty(num_chunks(sl, L), np.uint8)
    z32 = np.empty((T, 3), np.float32)
    z64 = np.empty((T, 3), np.float64)
    b3c = _c(b3, np.float32) if b3 is not None else None
    lib().mqo_route(len(sl), _p(sl, _i32p), int(L), D, H, _p(C, _f32p), _p(W1, _f32p),
                    _p(W2, _f32p), _p(W3, _f32p), _p(b3c, _f32p) if b3c is not None else None,
                    int(bool(routing_freeze)), _p(te, _u8p), _p(ce, _u8p), _p(z32, _f32p),
                    _p(z64, _f64p))
    return ce, te, z32, z64


def similarity_route(seq_lens, L, C, u, tau_hi, tau_lo, routing_freeze=True):
    """Returns (chunk_expert, fp64 similarity per chunk)."""
    sl = _c(seq_lens, np.int32)
    C = _c(C, np.float32)
    u = _c(u, np.float32)
    D = C.shape[1]
    assert u.shape == (len(sl), D) and C.shape[0] == int(sl.sum())
    n = num_chunks(sl, L)
    ce = np.empty(n, np.uint8)
    sim = np.empty(n, np.float64)
    lib().mqo_similarity_route(len(sl), _p(sl, _i32p), int(L), D, _p(C, _f32p), _p(u, _f32p),
                               float(tau_hi), float(tau_lo), int(bool(routing_freeze)),
                               _p(ce, _u8p), _p(sim, _f64p))
    return ce, sim


def layout_bytes(seq_lens, L):
    sl = _c(seq_lens, np.int32)
    return int(lib().mqo_layout_bytes(len(sl), _p(sl, _i32p), int(L)))


def build_layout(Hkv, d, L, seq_lens, chunk_expert):
    """Returns (layout blob as uint8 array, packed bytes of one layer)."""
    sl = _c(seq_lens, np.int32)
    ce = _c(chunk_expert, np.uint8)
    n = layout_bytes(sl, L)
    blob = np.zeros(n, np.uint8)
    pb = lib().mqo_build_layout(len(sl), int(Hkv), int(d), int(L), _p(sl, _i32p), _p(ce, _u8p),
                                _p(blob, _u8p), n)
    return blob, int(pb)


def packed_bytes(Hkv, d, L, seq_lens, chunk_expert):
    sl = _c(seq_lens, np.int32)
    ce = _c(chunk_expert, np.uint8)
    return int(lib().mqo_packed_bytes(len(sl), int(Hkv), int(d), int(L), _p(sl, _i32p),
                                      _p(ce, _u8p)))


def quantize_group(x, bits):
    """Returns (codes[32] uint8, s fp32, mn fp32, s fp16 bits, mn fp16 bits)."""
    x = _c(x, np.float32)
    assert x.shape == (32,)
    codes = np.empty(32, np.uint8)
    s = np.empty(1, np.float32)
    mn = np.empty(1, np.float32)
    sh = np.empty(1, np.uint16)
    mh = np.empty(1, np.uint16)
    lib().mqo_quantize_group(_p(x, _f32p), int(bits), _p(codes, _u8p), _p(s, _f32p),
                             _p(mn, _f32p), _p(sh, _u16p), _p(mh, _u16p))
    return codes, s[0], mn[0], sh[0], mh[0]


def pack_codes(codes, bits):
    codes = _c(codes, np.uint8)
    out = np.empty(4 * bits, np.uint8)
    lib().mqo_pack_codes(_p(codes, _u8p), int(bits), _p(out, _u8p))
    return out


def unpack_codes(raw, bits):
    raw = _c(raw, np.uint8)
    out = np.empty(32, np.uint8)
    lib().mqo_unpack_codes(_p(raw, _u8p), int(bits), _p(out, _u8p))
    return out


def pack(Hkv, d, L, seq_lens, chunk_expert, K, V, fill=0):
    """Packs one layer; K, V are [T, Hkv, d] float32 or float16 arrays."""
    sl = _c(seq_lens, np.int32)
    ce = _c(chunk_expert, np.uint8)
    assert K.dtype == V.dtype
    K = np.ascontiguousarray(K)
    V = np.ascontiguousarray(V)
    nbytes = packed_bytes(Hkv, d, L, sl, ce)
    out = np.full(nbytes, fill, np.uint8)
    rc = lib().mqo_pack(len(sl), int(Hkv), int(d), int(L), _p(sl, _i32p), _p(ce, _u8p),
                        K.ctypes.data, V.ctypes.data, _dtype_code(K), _p(out, _u8p), nbytes)
    assert rc == 0
    return out


def decode(Hq, Hkv, d, L, seq_lens, chunk_expert, packed, q, scale=0.0):
    """fp64 attention over this oracle's own packed layer; out [B, Hq, d]."""
    sl = _c(seq_lens, np.int32)
    ce = _c(chunk_expert, np.uint8)
    packed = _c(packed, np.uint8)
    q = np.ascontiguousarray(q)
    B = len(sl)
    out = np.empty((B, Hq, d), np.float64)
    lib().mqo_decode(B, int(Hq), int(Hkv), int(d), int(L), _p(sl, _i32p), _p(ce, _u8p),
                     _p(packed, _u8p), q.ctypes.data, _dtype_code(q), float(scale),
                     _p(out, _f64p))
    return out



def decode_partial(Hq, Hkv, d, L, seq_lens, chunk_expert, packed, q, scale=0.0):
    """decode plus (m, l) per (b, h): out [B, Hq, d], ml [B, Hq, 2] (fp64)."""
    sl = _c(seq_lens, np.int32)
    ce = _c(chunk_expert, np.uint8)
    packed = _c(packed, np.uint8)
    q = np.ascontiguousarray(q)
    B = len(sl)
    out = np.empty((B, Hq, d), np.float64)
    ml = np.empty((B, Hq, 2), np.float64)
    lib().mqo_decode_partial(B, int(Hq), int(Hkv), int(d), int(L), _p(sl, _i32p), _p(ce, _u8p),
                             _p(packed, _u8p), q.ctypes.data, _dtype_code(q), float(scale),
                             _p(out, _f64p), _p(ml, _f64p))
    return out, ml

def decode_pairs(Hq, Hkv, d, L, seq_lens, chunk_expert, K, V, q, pairs, scale=0.0):
    """fp64 attention for selected (b, h) pairs from raw K/V; out [n, d]."""
    sl = _c(seq_lens, np.int32)
    ce = _c(chunk_expert, np.uint8)
    K = np.ascontiguousarray(K)
    V = np.ascontiguousarray(V)
    q = np.ascontiguousarray(q)
    pr = _c(pairs, np.int32).reshape(-1, 2)
    out = np.empty((pr.shape[0], d), np.float64)
    lib().mqo_decode_pairs(len(sl), int(Hq), int(Hkv), int(d), int(L), _p(sl, _i32p),
                           _p(ce, _u8p), K.ctypes.data, V.ctypes.data, _dtype_code(K),
                           q.ctypes.data, _dtype_code(q), float(scale), _p(pr, _i32p),
                           pr.shape[0], _p(out, _f64p))
    return out


def dense_attention(Hq, Hkv, d, seq_lens, K, V, q, scale=0.0):
    sl = _c(seq_lens, np.int32)
    K = np.ascontiguousarray(K)
    V = np.ascontiguousarray(V)
    q = np.ascontiguousarray(q)
    B = len(sl)
    out = np.empty((B, Hq, d), np.float64)
    lib().mqo_dense_attention(B, int(Hq), int(Hkv), int(d), _p(sl, _i32p), K.ctypes.data,
                              V.ctypes.data, _dtype_code(K), q.ctypes.data, _dtype_code(q),
                              float(scale), _p(out, _f64p))
    return out


def f32_to_f16(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().mqo_f32_to_f16(_p(x, _f32p), _p(out, _u16p), x.size)
    return out.view(np.float16)


# layout-table field offsets, as the public header lays them out
HEADER_BYTES = 64
SEQ_BYTES = 160


def parse_layout(blob, B):
    """Splits a layout blob into (header dict, list of per-sequence dicts, perm, inv)."""
    blob = np.asarray(blob, np.uint8)
    hb = blob[:HEADER_BYTES]
    h = {
        "magic": int(hb[0:4].view(np.uint32)[0]),
        "version": int(hb[4:8].view(np.uint32)[0]),
        "num_seqs": int(hb[8:12].view(np.int32)[0]),
        "num_kv_heads": int(hb[12:16].view(np.int32)[0]),
        "head_dim": int(hb[16:20].view(np.int32)[0]),
        "chunk_len": int(hb[20:24].view(np.int32)[0]),
        "total_chunks": int(hb[24:28].view(np.int32)[0]),
        "total_items": int(hb[28:32].view(np.int32)[0]),
        "total_tokens": int(hb[32:40].view(np.int64)[0]),
        "packed_bytes": int(hb[40:48].view(np.uint64)[0]),
        "item_tokens": hb[48:60].view(np.int32).tolist(),
    }
    seqs = []
    for b in range(B):
        r = blob[HEADER_BYTES + b * SEQ_BYTES: HEADER_BYTES + (b + 1) * SEQ_BYTES]
        seqs.append({
            "token_offset": int(r[0:8].view(np.int64)[0]),
            "num_tokens": int(r[8:12].view(np.int32)[0]),
            "num_chunks": int(r[12:16].view(np.int32)[0]),
            "chunk_offset": int(r[16:20].view(np.int32)[0]),
            "seg_chunks": r[20:32].view(np.int32).tolist(),
            "seg_chunk_begin": r[32:44].view(np.int32).tolist(),
            "seg_tokens": r[44:56].view(np.int32).tolist(),
            "seg_base": r[56:80].view(np.uint64).tolist(),
            "region_bytes": r[80:104].view(np.uint64).tolist(),
            "scale_offset": r[104:128].view(np.uint64).tolist(),
            "item_begin": r[128:140].view(np.int32).tolist(),
            "item_count": r[140:152].view(np.int32).tolist(),
        })
    N = h["total_chunks"]
    p0 = HEADER_BYTES + B * SEQ_BYTES
    perm = blob[p0:p0 + 4 * N].view(np.int32).copy()
    p1 = p0 + ((4 * N + 15) // 16) * 16
    inv = blob[p1:p1 + 4 * N].view(np.int32).copy()
    return h, seqs, perm, inv
