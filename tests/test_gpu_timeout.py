"""Failure detection on the GPU without a fault: a bounded wait made to run
out through the test hook of include/mqkv_debug.h (a stage whose arrival is
withheld, a short wait bound).  The launch must stop, report
MQ_DEV_WAIT_TIMEOUT through the device status word, and leave the context
usable: the next call, unarmed, matches the oracle."""
import numpy as np
import pytest
import torch

from chunk_adaptive_mixed_b200 import mqkv as M
from oracle import oracle as O

from .gpu_helpers import Case, check_route, dev, gpu_route

pytestmark = pytest.mark.gpu


def _router_inputs(case, D, H, seed):
    g = torch.Generator().manual_seed(seed)
    C = torch.randn(case.T, D, generator=g)
    W1 = torch.randn(D, H, generator=g) / D ** 0.5
    W2 = torch.randn(D, H, generator=g) / D ** 0.5
    W3 = torch.randn(H, 3, generator=g) / H ** 0.5
    b3 = torch.tensor([0.0, 0.1, -0.05])
    return C, W1, W2, W3, b3


@pytest.mark.parametrize("H,D", [(128, 512), (64, 256)])
def test_router_wait_timeout_is_reported_and_the_context_stays_usable(H, D):
    lens = np.array([300, 64, 129], np.int32)
    case = Case(lens, 4, 4, 64, 64)
    C, W1, W2, W3, b3 = _router_inputs(case, D, H, seed=H + D)
    args = [x.to(dev()) for x in (C, W1, W2, W3, b3)]
    shp = case.shape()
    te = torch.empty(max(case.T, 16), dtype=torch.uint8, device=dev())
    ce = torch.empty(max(case.N, 16), dtype=torch.uint8, device=dev())
    ws = torch.empty(M.mq_route_workspace_bytes(shp, case.lens, D, H), dtype=torch.uint8,
                     device=dev())
    assert M.mq_device_status() == 0
    M.mq_debug_arm_wait_timeout(M.MQ_DEBUG_ROUTER)
    M.mq_route_chunks(shp, case.lens, case.cu(), *args, te, ce, ws)
    torch.cuda.synchronize()
    status = M.mq_device_status()
    assert status & M.MQ_DEV_WAIT_TIMEOUT, hex(status)
    # the arming was used up: the same call now runs normally and is right
    te2, ce2, logits = gpu_route(case, *args)
    z32, z64 = O.router_logits(C.numpy(), W1.numpy(), W2.numpy(), W3.numpy(), b3.numpy())
    check_route(lens, case.L, te2, ce2, logits, z32, z64, True)
