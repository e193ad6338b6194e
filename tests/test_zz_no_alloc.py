"""mq_decode_attn_noalloc: decode attention for callers that cannot allocate.

Callers such as a serving runtime that has reserved nearly all device memory
for its own pool, or a C program without a device allocator, cannot provide
the workspace mq_decode_attn needs; this entry point uses a scratch array
built into the library instead.  The GPU test checks, through the C ABI, that
two calls in a row give the same outputs as the workspace version: bit for
bit, since both run the same kernels on the same inputs and only the
workspace address differs (each work item's partial result is computed by
one warp in a fixed order and the merge visits the items in a fixed order,
so which warp takes which item does not change any bit).  It also checks the
outputs against the oracle within the attention tolerance of the other
tests.  This file is named so that it is collected last.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from chunk_adaptive_mixed_b200 import build as Bld
from chunk_adaptive_mixed_b200 import mqkv as M
from chunk_adaptive_mixed_b200 import workloads as W
from oracle import oracle as O

REL_L2 = 1e-3
MAX_ABS = 4e-3


def _close(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    return rel <= REL_L2 and np.abs(a - b).max() <= MAX_ABS


def test_scratch_size_matches_header():
    # the binding's copy of the scratch size is the header's value
    hdr = os.path.join(os.path.dirname(__file__), "..", "include", "mqkv.h")
    with open(hdr) as f:
        m = re.search(r"#define\s+MQ_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", f.read())
    assert m, "MQ_NOALLOC_SCRATCH_BYTES not found in include/mqkv.h"
    assert int(m.group(1)) << int(m.group(2)) == M.MQ_NOALLOC_SCRATCH_BYTES


def test_invalid_arguments_report_as_workspace_version():
    # runs without a GPU: argument checks come before any CUDA call, and the
    # no-allocation entry point reports them exactly as mq_decode_attn does
    Bld.build()
    p = 1 << 20
    cases = [
        (M.shape(2, 6, 4, 128, 128), np.array([100, 50], np.int32)),   # Hq % Hkv != 0
        (M.shape(2, 8, 4, 96, 128), np.array([100, 50], np.int32)),    # head_dim 96
        (M.shape(2, 8, 4, 128, 100), np.array([100, 50], np.int32)),   # chunk_len 100
        (M.shape(2, 8, 4, 128, 128), np.array([100, -5], np.int32)),   # negative length
    ]
    for shp, lens in cases:
        st_ws = M.lib().mq_decode_attn(ctypes.byref(shp), lens.ctypes.data, p, p, p, M.MQ_F16,
                                       0.0, p, 0, 0, 0)
        msg_ws = M.last_error()
        st_na = M.lib().mq_decode_attn_noalloc(ctypes.byref(shp), lens.ctypes.data, p, p, p,
                                               M.MQ_F16, 0.0, p, 0)
        msg_na = M.last_error()
        assert st_ws in (M.MQ_ERR_INVALID_ARG, M.MQ_ERR_UNSUPPORTED)
        assert (st_na, msg_na) == (st_ws, msg_ws)


def test_oversized_request_is_rejected_before_launch():
    # runs without a GPU: the size check happens on the host, first
    Bld.build()
    lens = np.array([32768] * 4, np.int32)
    shp = M.shape(4, 32, 32, 128, 128)
    assert M.mq_decode_workspace_bytes(shp, lens) > M.MQ_NOALLOC_SCRATCH_BYTES
    p = 1 << 20
    st = M.lib().mq_decode_attn_noalloc(ctypes.byref(shp), lens.ctypes.data, p, p, p, M.MQ_F16,
                                        0.0, p, 0)
    assert st == M.MQ_ERR_WORKSPACE
    assert "MQ_NOALLOC_SCRATCH_BYTES" in M.last_error()


@pytest.mark.gpu
def test_noalloc_matches_workspace_version_twice():
    Bld.build()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    lens = np.array([3000, 1, 0, 777, 129], np.int32)
    B, Hq, Hkv, d, L = len(lens), 16, 4, 128, 128
    shp = M.shape(B, Hq, Hkv, d, L)
    assert M.mq_decode_workspace_bytes(shp, lens) <= M.MQ_NOALLOC_SCRATCH_BYTES
    g = torch.Generator().manual_seed(123)
    T = int(lens.sum())
    K = torch.randn(T, Hkv, d, generator=g).half().to(dev)
    V = torch.randn(T, Hkv, d, generator=g).half().to(dev)
    q1 = torch.randn(B, Hq, d, generator=g).half().to(dev)
    q2 = torch.randn(B, Hq, d, generator=g).half().to(dev)
    cmap = W.synthetic_chunk_map(lens, L, mix=(0.2, 0.5, 0.3), seed=7)
    cu = torch.as_tensor(W.cu_seqlens(lens), device=dev)
    ce = torch.as_tensor(np.concatenate([cmap, np.zeros(16, np.uint8)]), device=dev)
    layout = torch.empty(M.mq_layout_bytes(shp, lens), dtype=torch.uint8, device=dev)
    M.mq_build_layout(shp, lens, cu, ce, layout)
    packed = torch.empty(M.mq_packed_bytes(layout), dtype=torch.uint8, device=dev)
    M.mq_pack_kv(shp, lens, layout, K, V, packed)
    ws = torch.empty(M.mq_decode_workspace_bytes(shp, lens), dtype=torch.uint8, device=dev)
    packed_o = O.pack(Hkv, d, L, lens, cmap, K.cpu().numpy(), V.cpu().numpy())
    for q in (q1, q2):  # two calls in a row, different queries
        ref = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
        got = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device=dev)
        M.mq_decode_attn(shp, lens, layout, packed, q, ref, ws)
        M.mq_decode_attn_noalloc(shp, lens, layout, packed, q, got)
        torch.cuda.synchronize()
        assert M.mq_device_status() == 0
        assert torch.equal(got, ref)
        want = O.decode(Hq, Hkv, d, L, lens, cmap, packed_o, q.cpu().numpy())
        assert _close(got.cpu().numpy(), want)
