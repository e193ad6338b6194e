"""Thin Python binding of libmqkv (include/mqkv.h).

Argument marshalling only: every function forwards to the C entry point of the
same name, passing raw device pointers taken from torch tensors and the
current (or given) CUDA stream.  Nothing here computes any step of the path,
and there is no fallback: if libmqkv.so is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmqkv.so")

MQ_OK = 0
MQ_ERR_INVALID_ARG = 1
MQ_ERR_UNSUPPORTED = 2
MQ_ERR_WORKSPACE = 3
MQ_ERR_CUDA = 4
MQ_ERR_DEVICE_CHECK = 5

MQ_F32 = 0
MQ_F16 = 1

MQ_DEV_PACKED_TOO_SMALL = 0x1
MQ_DEV_WORKSPACE_TOO_SMALL = 0x2
MQ_DEV_BAD_LAYOUT = 0x4
MQ_DEV_WAIT_TIMEOUT = 0x8
MQ_DEV_INDEX_RANGE = 0x10
MQ_DEV_CAPACITY = 0x20
MQ_GROW_OPEN = 0x1
MQ_GROW_FULL = 0x2

# test hook targets (include/mqkv_debug.h)
MQ_DEBUG_ROUTER = 0x1

# names of every function include/*.h declares
EXPORTS = ("mq_status_string", "mq_last_error", "mq_layout_bytes", "mq_packed_bytes_upper_bound",
           "mq_decode_workspace_bytes", "mq_route_workspace_bytes", "mq_packed_bytes", "mq_device_status", "mq_route_chunks",
           "mq_similarity_route", "mq_build_layout", "mq_pack_kv", "mq_decode_attn", "mq_decode_attn_noalloc",
           "mq_grow_sizes", "mq_grow_build_layout", "mq_grow_pack_kv", "mq_grow_commit",
           "mq_grow_append_kv", "mq_grow_seal", "mq_decode_attn_partial", "mq_combine_partials",
           "mq_debug_arm_wait_timeout")

# size of the scratch array built into the library for mq_decode_attn_noalloc
MQ_NOALLOC_SCRATCH_BYTES = 16 << 20


class MqShape(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("chunk_len", ctypes.c_int32), ("group_size", ctypes.c_int32)]


def shape(num_seqs, num_q_heads, num_kv_heads, head_dim, chunk_len, group_size=32) -> MqShape:
    return MqShape(num_seqs, num_q_heads, num_kv_heads, head_dim, chunk_len, group_size)


class MqkvError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libmqkv.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m chunk_adaptive_mixed_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, i32, u32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.POINTER(ctypes.c_uint32)
    sp = ctypes.POINTER(MqShape)
    L.mq_status_string.restype = ctypes.c_char_p
    L.mq_status_string.argtypes = [ctypes.c_int]
    L.mq_last_error.restype = ctypes.c_char_p
    L.mq_last_error.argtypes = []
    for name in ("mq_layout_bytes", "mq_packed_bytes_upper_bound", "mq_decode_workspace_bytes"):
        f = getattr(L, name)
        f.restype = sz
        f.argtypes = [sp, vp]
    L.mq_packed_bytes.restype = ctypes.c_int
    L.mq_packed_bytes.argtypes = [vp, ctypes.POINTER(ctypes.c_size_t), vp]
    L.mq_device_status.restype = ctypes.c_int
    L.mq_device_status.argtypes = [u32p, i32, vp]
    L.mq_route_workspace_bytes.restype = sz
    L.mq_route_workspace_bytes.argtypes = [sp, vp, i32, i32]
    L.mq_route_chunks.restype = ctypes.c_int
    L.mq_route_chunks.argtypes = [sp, vp, vp, vp, i32, i32, vp, vp, vp, vp, i32, vp, vp, vp, vp,
                                  sz, vp]
    L.mq_similarity_route.restype = ctypes.c_int
    L.mq_similarity_route.argtypes = [sp, vp, vp, vp, i32, vp, ctypes.c_double, ctypes.c_double,
                                      i32, vp, vp, vp]
    L.mq_build_layout.restype = ctypes.c_int
    L.mq_build_layout.argtypes = [sp, vp, vp, vp, vp, sz, vp]
    szp = ctypes.POINTER(ctypes.c_size_t)
    L.mq_grow_sizes.restype = ctypes.c_int
    L.mq_grow_sizes.argtypes = [sp, vp, i32, szp, szp, szp]
    L.mq_grow_build_layout.restype = ctypes.c_int
    L.mq_grow_build_layout.argtypes = [sp, vp, i32, vp, vp, vp, sz, vp]
    L.mq_grow_pack_kv.restype = ctypes.c_int
    L.mq_grow_pack_kv.argtypes = [sp, vp, i32, vp, vp, vp, i32, vp, sz, vp]
    L.mq_grow_commit.restype = ctypes.c_int
    L.mq_grow_commit.argtypes = [sp, vp, vp, i32, vp]
    L.mq_grow_append_kv.restype = ctypes.c_int
    L.mq_grow_append_kv.argtypes = [sp, vp, vp, vp, i32, vp, sz, vp]
    L.mq_grow_seal.restype = ctypes.c_int
    L.mq_grow_seal.argtypes = [sp, vp, vp, vp, sz, vp]
    L.mq_decode_attn_partial.restype = ctypes.c_int
    L.mq_decode_attn_partial.argtypes = [sp, vp, vp, vp, vp, i32, ctypes.c_float, vp, vp, sz, vp]
    L.mq_combine_partials.restype = ctypes.c_int
    L.mq_combine_partials.argtypes = [i32, i32, i32, i32, vp, vp, vp]
    L.mq_pack_kv.restype = ctypes.c_int
    L.mq_pack_kv.argtypes = [sp, vp, vp, vp, vp, i32, vp, sz, vp]
    L.mq_decode_attn.restype = ctypes.c_int
    L.mq_decode_attn.argtypes = [sp, vp, vp, vp, vp, i32, ctypes.c_float, vp, vp, sz, vp]
    L.mq_decode_attn_noalloc.restype = ctypes.c_int
    L.mq_decode_attn_noalloc.argtypes = [sp, vp, vp, vp, vp, i32, ctypes.c_float, vp, vp]
    _lib = L
    return L


def last_error() -> str:
    return lib().mq_last_error().decode()


def status_string(st: int) -> str:
    return lib().mq_status_string(st).decode()


def _check(st: int, what: str):
    if st != MQ_OK:
        raise MqkvError(st, f"{what}: {status_string(st)}: {last_error()}")


def _ptr(t) -> Optional[int]:
    """Raw pointer of a torch tensor / numpy array / int / None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _lens(seq_lens) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    return a


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return MQ_F16
    if t.dtype == torch.float32:
        return MQ_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---------------------------------------------------------------- size queries

def mq_layout_bytes(shp: MqShape, seq_lens: Sequence[int]) -> int:
    l = _lens(seq_lens)
    n = lib().mq_layout_bytes(ctypes.byref(shp), l.ctypes.data)
    if n == 0:
        raise MqkvError(MQ_ERR_INVALID_ARG, last_error())
    return int(n)


def mq_packed_bytes_upper_bound(shp: MqShape, seq_lens: Sequence[int]) -> int:
    l = _lens(seq_lens)
    return int(lib().mq_packed_bytes_upper_bound(ctypes.byref(shp), l.ctypes.data))


def mq_decode_workspace_bytes(shp: MqShape, seq_lens: Sequence[int]) -> int:
    l = _lens(seq_lens)
    n = lib().mq_decode_workspace_bytes(ctypes.byref(shp), l.ctypes.data)
    if n == 0:
        raise MqkvError(MQ_ERR_INVALID_ARG, last_error())
    return int(n)


def mq_packed_bytes(layout, stream=None) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().mq_packed_bytes(_ptr(layout), ctypes.byref(out), _stream(stream)),
           "mq_packed_bytes")
    return int(out.value)


def mq_device_status(clear: bool = True, stream=None) -> int:
    """Returns the device status bits (MQ_DEV_*) and clears them by default."""
    flags = ctypes.c_uint32(0)
    st = lib().mq_device_status(ctypes.byref(flags), int(bool(clear)), _stream(stream))
    if st not in (MQ_OK, MQ_ERR_DEVICE_CHECK):
        _check(st, "mq_device_status")
    return int(flags.value)


def mq_debug_arm_wait_timeout(kernels: int) -> None:
    """Test hook: the next launch of each named kernel (MQ_DEBUG_*) stops at
    a withheld stage through its bounded wait and sets MQ_DEV_WAIT_TIMEOUT."""
    L = lib()
    L.mq_debug_arm_wait_timeout.restype = ctypes.c_int
    L.mq_debug_arm_wait_timeout.argtypes = [ctypes.c_uint32]
    _check(L.mq_debug_arm_wait_timeout(int(kernels)), "mq_debug_arm_wait_timeout")


# ---------------------------------------------------------------- the path

def mq_route_workspace_bytes(shp, seq_lens, D, H) -> int:
    l = _lens(seq_lens)
    n = lib().mq_route_workspace_bytes(ctypes.byref(shp), l.ctypes.data, int(D), int(H))
    if n == 0:
        raise MqkvError(MQ_ERR_INVALID_ARG, last_error())
    return int(n)


def mq_route_chunks(shp, seq_lens, cu_seqlens, C, W1, W2, W3, b3, token_expert, chunk_expert,
                    workspace, logits=None, routing_freeze=True, stream=None):
    l = _lens(seq_lens)
    D, H = int(C.shape[1]), int(W1.shape[1])
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().mq_route_chunks(ctypes.byref(shp), l.ctypes.data, _ptr(cu_seqlens), _ptr(C), D, H,
                                 _ptr(W1), _ptr(W2), _ptr(W3), _ptr(b3), int(bool(routing_freeze)),
                                 _ptr(token_expert), _ptr(chunk_expert), _ptr(logits),
                                 _ptr(workspace), nbytes, _stream(stream)), "mq_route_chunks")


def mq_similarity_route(shp, seq_lens, cu_seqlens, C, u, tau_hi, tau_lo, chunk_expert,
                        similarity=None, routing_freeze=True, stream=None):
    l = _lens(seq_lens)
    _check(lib().mq_similarity_route(ctypes.byref(shp), l.ctypes.data, _ptr(cu_seqlens), _ptr(C),
                                     int(C.shape[1]), _ptr(u), float(tau_hi), float(tau_lo),
                                     int(bool(routing_freeze)), _ptr(chunk_expert),
                                     _ptr(similarity), _stream(stream)), "mq_similarity_route")


def mq_build_layout(shp, seq_lens, cu_seqlens, chunk_expert, layout, stream=None):
    l = _lens(seq_lens)
    nbytes = layout.numel() * layout.element_size()
    _check(lib().mq_build_layout(ctypes.byref(shp), l.ctypes.data, _ptr(cu_seqlens),
                                 _ptr(chunk_expert), _ptr(layout), nbytes, _stream(stream)),
           "mq_build_layout")


def mq_pack_kv(shp, seq_lens, layout, K, V, packed, stream=None):
    l = _lens(seq_lens)
    nbytes = packed.numel() * packed.element_size()
    _check(lib().mq_pack_kv(ctypes.byref(shp), l.ctypes.data, _ptr(layout), _ptr(K), _ptr(V),
                            _dtype_code(K), _ptr(packed), nbytes, _stream(stream)), "mq_pack_kv")


def mq_decode_attn(shp, seq_lens, layout, packed, q, out, workspace, softmax_scale=0.0,
                   stream=None):
    l = _lens(seq_lens)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().mq_decode_attn(ctypes.byref(shp), l.ctypes.data, _ptr(layout), _ptr(packed),
                                _ptr(q), _dtype_code(q), float(softmax_scale), _ptr(out),
                                _ptr(workspace), nbytes, _stream(stream)), "mq_decode_attn")


def mq_decode_attn_noalloc(shp, seq_lens, layout, packed, q, out, softmax_scale=0.0, stream=None):
    """mq_decode_attn using the library's built-in scratch array instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    l = _lens(seq_lens)
    _check(lib().mq_decode_attn_noalloc(ctypes.byref(shp), l.ctypes.data, _ptr(layout),
                                        _ptr(packed), _ptr(q), _dtype_code(q),
                                        float(softmax_scale), _ptr(out), _stream(stream)),
           "mq_decode_attn_noalloc")


# ------------------------------------------------------------------ growth

def mq_grow_sizes(shp, seq_lens, grow_tokens):
    """(layout bytes, packed-bytes upper bound, decode workspace bytes)."""
    l = _lens(seq_lens)
    a, b, c = ctypes.c_size_t(0), ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib().mq_grow_sizes(ctypes.byref(shp), l.ctypes.data, int(grow_tokens),
                               ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)), "mq_grow_sizes")
    return a.value, b.value, c.value


def mq_grow_build_layout(shp, seq_lens, grow_tokens, cu_seqlens, chunk_expert, layout,
                         stream=None):
    l = _lens(seq_lens)
    nbytes = layout.numel() * layout.element_size()
    _check(lib().mq_grow_build_layout(ctypes.byref(shp), l.ctypes.data, int(grow_tokens),
                                      _ptr(cu_seqlens), _ptr(chunk_expert), _ptr(layout), nbytes,
                                      _stream(stream)), "mq_grow_build_layout")


def mq_grow_pack_kv(shp, seq_lens, grow_tokens, layout, K, V, packed, stream=None):
    l = _lens(seq_lens)
    nbytes = packed.numel() * packed.element_size()
    _check(lib().mq_grow_pack_kv(ctypes.byref(shp), l.ctypes.data, int(grow_tokens), _ptr(layout),
                                 _ptr(K), _ptr(V), _dtype_code(K), _ptr(packed), nbytes,
                                 _stream(stream)), "mq_grow_pack_kv")


def mq_grow_commit(shp, layout, sealed=None, add_token=True, stream=None):
    _check(lib().mq_grow_commit(ctypes.byref(shp), _ptr(layout), _ptr(sealed),
                                int(bool(add_token)), _stream(stream)), "mq_grow_commit")


def mq_grow_append_kv(shp, layout, K_new, V_new, packed, stream=None):
    nbytes = packed.numel() * packed.element_size()
    _check(lib().mq_grow_append_kv(ctypes.byref(shp), _ptr(layout), _ptr(K_new), _ptr(V_new),
                                   _dtype_code(K_new), _ptr(packed), nbytes, _stream(stream)),
           "mq_grow_append_kv")


def mq_grow_seal(shp, layout, sealed, packed, stream=None):
    nbytes = packed.numel() * packed.element_size()
    _check(lib().mq_grow_seal(ctypes.byref(shp), _ptr(layout), _ptr(sealed), _ptr(packed), nbytes,
                              _stream(stream)), "mq_grow_seal")


# ------------------------------------------------------------ context split

def partial_floats(head_dim: int) -> int:
    """Floats of one (sequence, head) record of mq_decode_attn_partial."""
    return head_dim + 4


def mq_decode_attn_partial(shp, seq_lens, layout, packed, q, partial, workspace,
                           softmax_scale=0.0, stream=None):
    l = _lens(seq_lens)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().mq_decode_attn_partial(ctypes.byref(shp), l.ctypes.data, _ptr(layout),
                                        _ptr(packed), _ptr(q), _dtype_code(q),
                                        float(softmax_scale), _ptr(partial), _ptr(workspace),
                                        nbytes, _stream(stream)), "mq_decode_attn_partial")


def mq_combine_partials(partials, out, stream=None):
    """partials [P, B, Hq, d + 4] fp32 -> out [B, Hq, d] fp32."""
    P, B, Hq, rec = partials.shape
    _check(lib().mq_combine_partials(int(P), int(B), int(Hq), int(rec - 4), _ptr(partials),
                                     _ptr(out), _stream(stream)), "mq_combine_partials")
