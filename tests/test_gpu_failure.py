"""Failure detection on the GPU without a fault: a bounded device-side wait that
nothing completes gives up, records its code in the workspace status word and
returns; the host reads DMA_ERR_TIMEOUT, clears the word, and the same context
and workspace then compute a correct forward."""
import ctypes

import numpy as np
import pytest

import oracle
from workloads import get, make_inputs

from gpu_common import assert_close, lib, to_dev, to_np, torch_cuda

pytestmark = pytest.mark.gpu

DMA_ERR_TIMEOUT = 5


def test_bounded_wait_gives_up_reports_and_leaves_the_context_usable():
    dma = lib()
    torch = torch_cuda()
    wl = get("tiny").with_(dtype="bf16", d=128, seed=81)
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, dtype=wl.dtype)
    ws = dma.alloc_workspace(p)
    assert dma.check_device_status(p, ws) == 0
    dma.selftest_bounded_wait(p, ws, 2_000_000)   # about a millisecond of SM clock
    code = ctypes.c_int32(0)
    st = dma.load().dma_check_device_status(ctypes.byref(p), ctypes.c_void_p(ws.data_ptr()), None, ctypes.byref(code))
    assert st == DMA_ERR_TIMEOUT and (code.value & 0x1)
    dma.clear_device_status(p, ws)
    assert dma.check_device_status(p, ws) == 0
    I = make_inputs(wl)
    r = dma.forward(p, to_dev(I.Q, I.bits.get("Q"), wl.dtype), to_dev(I.K, I.bits.get("K"), wl.dtype),
                    to_dev(I.V, I.bits.get("V"), wl.dtype), to_dev(I.Delta, I.bits.get("Delta"), wl.dtype),
                    torch.from_numpy(I.A).cuda(), workspace=ws)
    torch.cuda.synchronize()
    d32 = to_np(r["delta"])
    e = np.stack([np.stack([oracle.topw_eviction(d32[b, h], wl.w) for h in range(wl.H)]) for b in range(wl.B)])
    O_ref, L_ref = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e)
    assert_close(to_np(r["LSE"]), L_ref, "LSE")
    assert_close(to_np(r["O"]), O_ref, "O")
    assert dma.check_device_status(p, ws) == 0
