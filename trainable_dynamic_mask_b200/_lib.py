"""ctypes declarations of libdma's C ABI (include/dma.h).

Loading fails loudly when the library has not been built: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdma.so")

c_i32 = ctypes.c_int32
c_f32 = ctypes.c_float
c_vp = ctypes.c_void_p
c_sz = ctypes.c_size_t

DMA_OK = 0
STATUS_NAMES = {0: "DMA_OK", 1: "DMA_ERR_INVALID_ARG", 2: "DMA_ERR_UNSUPPORTED",
                3: "DMA_ERR_WORKSPACE", 4: "DMA_ERR_CUDA", 5: "DMA_ERR_TIMEOUT"}
DMA_BF16 = 0
DMA_F32 = 1
DMA_FLAG_FORWARD_ONLY = 1
BLOCK_Q = 128
NOALLOC_SCRATCH_BYTES = 16 << 20


class DmaParams(ctypes.Structure):
    _fields_ = [("B", c_i32), ("H", c_i32), ("Hkv", c_i32), ("N", c_i32), ("Nq", c_i32),
                ("d", c_i32), ("w", c_i32), ("scale", c_f32), ("dtype", c_i32), ("flags", c_i32),
                ("w_heads", c_vp)]


class DmaWsLayout(ctypes.Structure):
    _fields_ = [("bytes", c_sz), ("off_status", c_sz), ("off_counts", c_sz), ("off_lists", c_sz),
                ("off_sel", c_sz), ("n_blocks", c_i32), ("list_cap", c_i32), ("sel_len", c_i32),
                ("reserved", c_i32)]


class DmaCpLayout(ctypes.Structure):
    _fields_ = [("cand_bytes", c_sz), ("off_pos", c_sz), ("off_delta", c_sz), ("off_k", c_sz), ("off_v", c_sz),
                ("ws_bytes", c_sz), ("off_status", c_sz), ("prefix_rows", c_i32), ("reserved", c_i32)]


# name -> argtypes (every function returns dma_status_t as int32 unless listed in _RESTYPES)
_SIGS = {
    "dma_status_string": [c_i32],
    "dma_abi_version": [],
    "dma_workspace_size": [ctypes.POINTER(DmaParams), ctypes.POINTER(c_sz)],
    "dma_workspace_layout": [ctypes.POINTER(DmaParams), ctypes.POINTER(DmaWsLayout)],
    "dma_gate": [ctypes.POINTER(DmaParams), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp],
    "dma_topk_mask": [ctypes.POINTER(DmaParams), c_vp, c_vp, c_vp, c_sz, c_vp],
    "dma_topk_append": [ctypes.POINTER(DmaParams), c_vp, c_vp, c_sz, c_vp],
    "dma_gate_append": [ctypes.POINTER(DmaParams), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp],
    "dma_attn_fwd": [ctypes.POINTER(DmaParams), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp, c_vp,
                     c_vp],
    "dma_attn_bwd": [ctypes.POINTER(DmaParams), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp, c_vp,
                     c_vp, c_vp, c_vp, c_vp, c_vp, c_vp],
    "dma_gate_bwd": [ctypes.POINTER(DmaParams), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                     c_vp, c_sz, c_vp],
    "dma_gate_bwd_noalloc": [ctypes.POINTER(DmaParams), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                             c_vp],
    "dma_check_device_status": [ctypes.POINTER(DmaParams), c_vp, c_vp, ctypes.POINTER(c_i32)],
    "dma_clear_device_status": [ctypes.POINTER(DmaParams), c_vp, c_vp],
    "dma_selftest_bounded_wait": [ctypes.POINTER(DmaParams), c_vp, c_sz, ctypes.c_int64, c_vp],
    "dma_cp_layout": [ctypes.POINTER(DmaParams), c_i32, c_i32, ctypes.POINTER(DmaCpLayout)],
    "dma_cp_candidates": [ctypes.POINTER(DmaParams), c_i32, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp, c_sz, c_vp],
    "dma_cp_compact": [ctypes.POINTER(DmaParams), c_i32, c_i32, c_vp, c_sz, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                       c_vp, c_sz, c_vp],
}
_RESTYPES = {"dma_status_string": ctypes.c_char_p, "dma_abi_version": c_i32}

_lib = None


def load() -> ctypes.CDLL:
    """Load libdma.so (built by `python -m trainable_dynamic_mask_b200.build`)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m trainable_dynamic_mask_b200.build`"
                " (there is no fallback implementation)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = _RESTYPES.get(name, c_i32)
        _lib = lib
    return _lib


def exported_names() -> list[str]:
    return list(_SIGS)


class DmaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        try:
            msg = load().dma_status_string(code).decode()
        except Exception:  # pragma: no cover - message lookup is best effort
            msg = STATUS_NAMES.get(code, str(code))
        super().__init__(f"{fn} failed: {msg}")


def check(fn: str, code: int) -> None:
    if code != DMA_OK:
        raise DmaError(fn, code)
