"""The workspace-free gate backward (dma_gate_bwd_noalloc), for callers that
cannot allocate device memory -- code running where cudaMalloc is off limits,
for instance inside a host application or framework that owns the GPU's
allocator.  Its scratch is a fixed array inside the library, so these tests
check that it gives the workspace entry point's results, and the oracle's gate
backward, on two calls in a row (the second call must not see stale scratch
from the first).  The refusal of a problem too large for the array, with the
scratch formula exact at its boundary, is checked on the host, without a GPU,
in test_abi.py.

This file is collected last on purpose: the GPU tests before it have all run
when it starts, and it also passes in a fresh process on its own."""
import numpy as np
import pytest

import oracle
from workloads import get, make_inputs

from gpu_common import assert_close, f32_dev, lib, to_dev, to_np, torch_cuda

pytestmark = pytest.mark.gpu


def _gate_inputs(dma, torch, wl, I):
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, dtype=wl.dtype)
    V = to_dev(I.V, I.bits.get("V"), wl.dtype)
    D = to_dev(I.Delta, I.bits.get("Delta"), wl.dtype)
    A = f32_dev(I.A)
    delta = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device="cuda")
    x = torch.empty_like(delta)
    dma.gate(p, V, D, A, delta, x)
    return p, V, D, A, delta, x


def _outputs(torch, wl):
    return (torch.full((wl.Hkv * wl.d, wl.H), float("nan"), dtype=torch.float32, device="cuda"),
            torch.full((wl.H,), float("nan"), dtype=torch.float32, device="cuda"),
            torch.full((wl.B, wl.Hkv, wl.N, wl.d), float("nan"), dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("wl", [get("prefill"), get("tiny").with_(B=2, H=6, Hkv=3, N=333, d=64, seed=61)],
                         ids=["prefill", "odd_f32"])
def test_noalloc_matches_workspace_entry_point_twice(wl):
    dma = lib()
    torch = torch_cuda()
    I = make_inputs(wl)
    p, V, D, A, delta, x = _gate_inputs(dma, torch, wl, I)
    ws = dma.alloc_workspace(p)
    rng = np.random.default_rng(wl.seed + 7)
    for call in range(2):
        g32 = rng.standard_normal((wl.B, wl.H, wl.N)).astype(np.float32)
        g = f32_dev(g32)
        ref = _outputs(torch, wl)
        dma.gate_bwd(p, V, D, A, x, delta, g, *ref, ws)
        got = _outputs(torch, wl)
        dma.gate_bwd_noalloc(p, V, D, A, x, delta, g, *got)
        torch.cuda.synchronize()
        orc = oracle.gate_bwd(I.V, I.Delta, I.A, g32.astype(np.float64))
        for name, a, b, o in zip(("dDelta", "dA", "dV_gate"), got, ref, orc):
            assert_close(to_np(a), to_np(b), f"{name} (call {call + 1}, against dma_gate_bwd)")
            assert_close(to_np(a), o, f"{name} (call {call + 1}, against the oracle)")
