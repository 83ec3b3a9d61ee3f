"""Shared helpers of the GPU parity tests (inputs to the device, tolerances).

Parity bar: the mask (eviction index, block lists, decode selection) is
compared bit for bit; delta within 1e-5 relative; O, LSE and gradients within
|gpu - oracle| <= 2e-2 + 1e-2 |oracle| (2e-2 max-abs, 1e-2 relative).
"""
from __future__ import annotations

import os

import numpy as np
import pytest

ATOL = 2e-2
RTOL = 1e-2
DELTA_RTOL = 1e-5


def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    return torch


def lib():
    import trainable_dynamic_mask_b200 as dma
    from trainable_dynamic_mask_b200 import _lib
    if not os.path.exists(_lib.LIB_PATH):
        from trainable_dynamic_mask_b200 import build
        build.build()
    dma.load()
    return dma


def to_dev(arr: np.ndarray, bits: np.ndarray | None, dtype: str):
    """Exact device copy of an input: bf16 bits when dtype == 'bf16', else float32."""
    torch = torch_cuda()
    if dtype == "bf16":
        assert bits is not None
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    return t.cuda().contiguous()


def f32_dev(a: np.ndarray):
    torch = torch_cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def to_np(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def assert_close(gpu, ref, name, atol=ATOL, rtol=RTOL):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (name, gpu.shape, ref.shape)
    assert np.isfinite(gpu).all(), f"{name}: non-finite GPU values"
    err = np.abs(gpu - ref)
    bad = err > atol + rtol * np.abs(ref)
    if bad.any():
        i = np.unravel_index(np.argmax(err - (atol + rtol * np.abs(ref))), err.shape)
        raise AssertionError(f"{name}: {int(bad.sum())} of {bad.size} outside tolerance; worst at {i}: "
                             f"gpu={gpu[i]!r} oracle={ref[i]!r} (max abs err {err.max():.3e})")


def assert_delta_close(gpu, ref, name="delta"):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rel = np.abs(gpu - ref) / np.abs(ref)
    assert rel.max() <= DELTA_RTOL, f"{name}: max relative error {rel.max():.3e}"
