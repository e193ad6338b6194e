"""The C ABI on a machine without a GPU: the library loads, exports every
function include/mqkv.h declares, validates arguments before touching CUDA,
and its size queries agree with the header's closed forms (checked through
the CPU oracle's independent implementation of the format)."""
import ctypes
import os
import re

import numpy as np
import pytest

from chunk_adaptive_mixed_b200 import build as B
from chunk_adaptive_mixed_b200 import mqkv as M
from oracle import oracle as O

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
HEADER = os.path.join(INCLUDE, "mqkv.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()
    yield


def declared_functions():
    # every header under include/ (the interface and its test hooks)
    text = "".join(open(os.path.join(INCLUDE, f)).read() for f in sorted(os.listdir(INCLUDE))
                   if f.endswith(".h"))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mq_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(M.EXPORTS)


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(M.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings():
    for st in range(6):
        assert M.status_string(st)
    assert M.status_string(99) == "unknown status"


def _shape(**kw):
    base = dict(num_seqs=2, num_q_heads=8, num_kv_heads=2, head_dim=128, chunk_len=64)
    base.update(kw)
    return M.shape(**base)


LENS = np.array([300, 64], np.int32)


@pytest.mark.parametrize("kw,status", [
    (dict(num_seqs=0), M.MQ_ERR_INVALID_ARG),
    (dict(num_q_heads=6, num_kv_heads=4), M.MQ_ERR_INVALID_ARG),
    (dict(num_q_heads=12, num_kv_heads=4), M.MQ_ERR_UNSUPPORTED),   # Hq/Hkv = 3
    (dict(head_dim=96), M.MQ_ERR_UNSUPPORTED),
    (dict(chunk_len=48), M.MQ_ERR_INVALID_ARG),
    (dict(chunk_len=16), M.MQ_ERR_INVALID_ARG),
    (dict(group_size=64), M.MQ_ERR_UNSUPPORTED),
])
def test_bad_shapes_are_rejected_before_any_launch(kw, status):
    lib = M.lib()
    shp = _shape(**kw)
    lens = np.array([300, 64], np.int32)
    dummy = 1 << 20  # aligned, never dereferenced
    st = lib.mq_pack_kv(ctypes.byref(shp), lens.ctypes.data, dummy, dummy, dummy, M.MQ_F16, dummy,
                        1 << 20, 0)
    assert st == status, M.last_error()
    assert M.last_error()
    assert lib.mq_layout_bytes(ctypes.byref(shp), lens.ctypes.data) == 0


def test_bad_pointers_and_sizes():
    lib = M.lib()
    shp = _shape()
    lens = LENS.copy()
    p = 1 << 20
    # null / misaligned device pointers
    assert lib.mq_pack_kv(ctypes.byref(shp), lens.ctypes.data, None, p, p, 1, p, 1 << 20, 0) \
        == M.MQ_ERR_INVALID_ARG
    assert "layout" in M.last_error()
    assert lib.mq_pack_kv(ctypes.byref(shp), lens.ctypes.data, p + 4, p, p, 1, p, 1 << 20, 0) \
        == M.MQ_ERR_INVALID_ARG
    assert "aligned" in M.last_error()
    # negative length
    bad = np.array([300, -1], np.int32)
    assert lib.mq_pack_kv(ctypes.byref(shp), bad.ctypes.data, p, p, p, 1, p, 1 << 20, 0) \
        == M.MQ_ERR_INVALID_ARG
    # wrong dtype code
    assert lib.mq_pack_kv(ctypes.byref(shp), lens.ctypes.data, p, p, p, 7, p, 1 << 20, 0) \
        == M.MQ_ERR_INVALID_ARG
    # router: H unsupported, D not a multiple of 4
    assert lib.mq_route_chunks(ctypes.byref(shp), lens.ctypes.data, p, p, 64, 96, p, p, p, None, 1,
                               p, p, None, p, 1 << 30, 0) == M.MQ_ERR_UNSUPPORTED
    assert lib.mq_route_chunks(ctypes.byref(shp), lens.ctypes.data, p, p, 66, 64, p, p, p, None, 1,
                               p, p, None, p, 1 << 30, 0) == M.MQ_ERR_INVALID_ARG
    # router workspace too small
    rws = lib.mq_route_workspace_bytes(ctypes.byref(shp), lens.ctypes.data, 64, 64)
    assert rws > 0
    assert lib.mq_route_chunks(ctypes.byref(shp), lens.ctypes.data, p, p, 64, 64, p, p, p, None, 1,
                               p, p, None, p, rws - 1, 0) == M.MQ_ERR_WORKSPACE
    assert lib.mq_route_workspace_bytes(ctypes.byref(shp), lens.ctypes.data, 64, 100) == 0
    # layout buffer too small
    need = lib.mq_layout_bytes(ctypes.byref(shp), lens.ctypes.data)
    assert lib.mq_build_layout(ctypes.byref(shp), lens.ctypes.data, p, p, p, need - 16, 0) \
        == M.MQ_ERR_WORKSPACE
    # decode workspace too small
    ws = lib.mq_decode_workspace_bytes(ctypes.byref(shp), lens.ctypes.data)
    assert ws > 0
    assert lib.mq_decode_attn(ctypes.byref(shp), lens.ctypes.data, p, p, p, 1, 0.0, p, p, ws - 1,
                              0) == M.MQ_ERR_WORKSPACE
    assert lib.mq_packed_bytes(None, None, 0) == M.MQ_ERR_INVALID_ARG
    assert lib.mq_device_status(None, 0, 0) == M.MQ_ERR_INVALID_ARG


def test_valid_call_without_gpu_reports_cuda_error():
    # no silent CPU path: with valid arguments and no device the call fails
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    lib = M.lib()
    shp = _shape()
    lens = LENS.copy()
    p = 1 << 20
    need = lib.mq_layout_bytes(ctypes.byref(shp), lens.ctypes.data)
    st = lib.mq_build_layout(ctypes.byref(shp), lens.ctypes.data, p, p, p, need, 0)
    assert st == M.MQ_ERR_CUDA, M.last_error()


@pytest.mark.parametrize("d,L", [(64, 32), (128, 64), (128, 256)])
def test_size_queries_match_the_format(d, L):
    rng = np.random.default_rng(d + L)
    lens = rng.integers(0, 2000, 5).astype(np.int32)
    shp = _shape(num_seqs=5, head_dim=d, chunk_len=L)
    n = int(((lens + L - 1) // L).sum())
    assert M.mq_layout_bytes(shp, lens) == O.layout_bytes(lens, L)
    assert M.mq_packed_bytes_upper_bound(shp, lens) == \
        O.packed_bytes(2, d, L, lens, np.zeros(n, np.uint8))
    ce = rng.integers(0, 3, n).astype(np.uint8)
    assert O.packed_bytes(2, d, L, lens, ce) <= M.mq_packed_bytes_upper_bound(shp, lens)


def test_similarity_route_validation():
    lib = M.lib()
    shp = _shape()
    lens = LENS.copy()
    p = 1 << 20
    nan = float("nan")
    f = lib.mq_similarity_route
    assert f(ctypes.byref(shp), lens.ctypes.data, p, p, 64, p, 0.1, 0.0, 1, p, None, 0) \
        == M.MQ_ERR_CUDA                                   # valid, but no device here
    assert f(ctypes.byref(shp), lens.ctypes.data, p, p, 66, p, 0.1, 0.0, 1, p, None, 0) \
        == M.MQ_ERR_INVALID_ARG
    assert f(ctypes.byref(shp), lens.ctypes.data, p, p, 64, p, nan, 0.0, 1, p, None, 0) \
        == M.MQ_ERR_INVALID_ARG
    assert "NaN" in M.last_error()
    assert f(ctypes.byref(shp), lens.ctypes.data, p, p, 64, None, 0.1, 0.0, 1, p, None, 0) \
        == M.MQ_ERR_INVALID_ARG
    assert f(ctypes.byref(shp), lens.ctypes.data, p, p, 64, p, 0.1, 0.0, 1, p, p + 8, 0) \
        == M.MQ_ERR_INVALID_ARG
    big = _shape(num_seqs=70000)
    many = np.full(70000, 1, np.int32)
    assert f(ctypes.byref(big), many.ctypes.data, p, p, 64, p, 0.1, 0.0, 1, p, None, 0) \
        == M.MQ_ERR_UNSUPPORTED


def test_grow_sizes_and_validation():
    shp = _shape(num_seqs=3, head_dim=128, chunk_len=64)
    lens = np.array([300, 256, 0], np.int32)
    lay, pk, ws = M.mq_grow_sizes(shp, lens, 100)
    G = (100 + 63) // 64
    n = (lens + 63) // 64
    slots = int(n.sum()) + 3 * (G + 1)
    pad16 = lambda x: (x + 15) // 16 * 16
    assert lay == 64 + 3 * 160 + 2 * pad16(4 * slots)
    # all present chunks at FP16 plus the reservations of the three segments
    a128 = lambda x: (x + 127) // 128 * 128
    want = 0
    for nb in n.tolist():
        want += 2 * 2 * (a128((nb + 1 + G) * 64 * 256)
                         + a128(G * 64 * 64) + a128(G * 64 * 16)
                         + a128(G * 64 * 32) + a128(G * 64 * 16))
    assert pk == want
    assert ws >= M.mq_decode_workspace_bytes(shp, lens)
    lib = M.lib()
    z = ctypes.c_size_t(0)
    assert lib.mq_grow_sizes(ctypes.byref(shp), lens.ctypes.data, -1, ctypes.byref(z), None,
                             None) == M.MQ_ERR_INVALID_ARG
    big = np.array([1 << 23, 0, 0], np.int32)
    assert lib.mq_grow_sizes(ctypes.byref(shp), big.ctypes.data, 1, ctypes.byref(z), None,
                             None) == M.MQ_ERR_UNSUPPORTED
    p = 1 << 20
    assert lib.mq_grow_commit(ctypes.byref(shp), p, None, 2, 0) == M.MQ_ERR_INVALID_ARG
    assert lib.mq_grow_commit(ctypes.byref(shp), p, p + 1, 1, 0) == M.MQ_ERR_INVALID_ARG
    assert lib.mq_grow_seal(ctypes.byref(shp), p, None, p, 1 << 20, 0) == M.MQ_ERR_INVALID_ARG
    assert lib.mq_grow_append_kv(ctypes.byref(shp), p, p, p, 5, p, 1 << 20, 0) \
        == M.MQ_ERR_INVALID_ARG
    need = lay
    assert lib.mq_grow_build_layout(ctypes.byref(shp), lens.ctypes.data, 100, p, p, p, need - 16,
                                    0) == M.MQ_ERR_WORKSPACE
    # valid arguments, no device: a CUDA error, never a silent CPU path
    assert lib.mq_grow_build_layout(ctypes.byref(shp), lens.ctypes.data, 100, p, p, p, need,
                                    0) == M.MQ_ERR_CUDA


def test_debug_hook_rejects_unknown_kernels():
    # host only: arming makes no CUDA call, and bits outside MQ_DEBUG_* are refused
    L = M.lib()
    L.mq_debug_arm_wait_timeout.restype = ctypes.c_int
    L.mq_debug_arm_wait_timeout.argtypes = [ctypes.c_uint32]
    assert L.mq_debug_arm_wait_timeout(0x80) == M.MQ_ERR_INVALID_ARG
    assert L.mq_debug_arm_wait_timeout(0) == M.MQ_OK



def test_headers_serve_plain_c_and_cxx_consumers(tmp_path):
    # the boundary is a C ABI: a C99 program (pedantic, warnings as errors)
    # includes the headers, links libmqkv and gets the binding's answers
    import shutil
    import subprocess
    root = os.path.dirname(INCLUDE)
    gcc, gxx = shutil.which("gcc"), shutil.which("g++")
    if gcc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(M.LIB_PATH)
    exe = str(tmp_path / "consumer")
    subprocess.run([gcc, "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", root,
                    os.path.join(root, "tests", "abi_c", "consumer.c"), "-o", exe,
                    "-L", libdir, "-lmqkv", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    got = dict(line.split() for line in out if line and line != "ok")
    assert "ok" in out
    shp = M.shape(3, 32, 8, 128, 128)
    lens = np.array([1000, 0, 4097], np.int32)
    assert int(got["layout_bytes"]) == M.mq_layout_bytes(shp, lens)
    assert int(got["packed_upper"]) == M.mq_packed_bytes_upper_bound(shp, lens)
    assert int(got["decode_ws"]) == M.mq_decode_workspace_bytes(shp, lens)
    if gxx is not None:
        for h in sorted(os.listdir(INCLUDE)):
            src = tmp_path / "h.cpp"
            src.write_text(f'#include "include/{h}"\nint main() {{ return 0; }}\n')
            subprocess.run([gxx, "-std=c++17", "-Wall", "-Wextra", "-Werror", "-I", root,
                            "-fsyntax-only", str(src)], check=True)
