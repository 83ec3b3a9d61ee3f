"""Dynamic Mask Attention hot path on B200 (sm_100a): Python binding of libdma.

Every function here marshals arguments and calls the C ABI declared in
include/dma.h; all computation runs in the library's CUDA kernels.  PyTorch is
used for device memory and streams only.  Functions raise DmaError when the
library returns a status other than DMA_OK.

Method: "Trainable Dynamic Mask Sparse Attention" (HF blog "dmattn"):
gate delta = exp(softplus(v Delta) A), causal top-w mask, masked attention
softmax(q k^T / sqrt(d) + m) v, with its backward.
"""
from __future__ import annotations

import ctypes

from ._lib import (BLOCK_Q, DMA_BF16, DMA_F32, DMA_FLAG_FORWARD_ONLY, DmaCpLayout, DmaError, DmaParams, DmaWsLayout,
                   LIB_PATH, check, exported_names, load)

__all__ = [
    "BLOCK_Q", "DMA_BF16", "DMA_F32", "DmaError", "DmaParams", "LIB_PATH", "load", "exported_names",
    "make_params", "workspace_size", "workspace_layout", "gate", "topk_mask", "topk_append", "gate_append",
    "attn_fwd", "attn_bwd",
    "gate_bwd", "gate_bwd_noalloc", "check_device_status", "clear_device_status", "selftest_bounded_wait",
    "abi_version", "alloc_workspace", "forward",
    "backward", "cp_layout", "cp_candidates", "cp_compact",
]


def make_params(B, H, Hkv, N, d, w, Nq=None, scale=0.0, dtype="bf16", w_heads=None,
                forward_only=False) -> DmaParams:
    """dma_params_t for a problem (Nq defaults to N; Nq=1 is decode).

    forward_only: no backward follows (DMA_FLAG_FORWARD_ONLY): the forward keeps
    nothing for it in the workspace.

    w_heads: None, or per-head windows as a device int32 tensor of H values (or its
    device address); w must then be the largest of them.  The caller keeps the
    tensor alive for as long as the parameters are used."""
    dt = {"bf16": DMA_BF16, "f32": DMA_F32}[dtype] if isinstance(dtype, str) else int(dtype)
    return DmaParams(B=B, H=H, Hkv=Hkv, N=N, Nq=N if Nq is None else Nq, d=d, w=w,
                     scale=float(scale), dtype=dt, flags=DMA_FLAG_FORWARD_ONLY if forward_only else 0,
                     w_heads=_ptr(w_heads))


def abi_version() -> int:
    return int(load().dma_abi_version())


def workspace_size(p: DmaParams) -> int:
    n = ctypes.c_size_t(0)
    check("dma_workspace_size", load().dma_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return int(n.value)


def workspace_layout(p: DmaParams) -> DmaWsLayout:
    lay = DmaWsLayout()
    check("dma_workspace_layout", load().dma_workspace_layout(ctypes.byref(p), ctypes.byref(lay)))
    return lay


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to libdma must be contiguous")
    return t.data_ptr()


def _nbytes(t):
    if t is None:
        return 0
    return t.numel() * t.element_size()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def gate(p, V, Delta, A, delta, x_save=None, workspace=None, stream=None):
    check("dma_gate", load().dma_gate(ctypes.byref(p), _ptr(V), _ptr(Delta), _ptr(A), _ptr(delta),
                                      _ptr(x_save), _ptr(workspace), _nbytes(workspace), _stream(stream)))


def topk_mask(p, delta, evict, workspace, stream=None):
    check("dma_topk_mask", load().dma_topk_mask(ctypes.byref(p), _ptr(delta), _ptr(evict),
                                                _ptr(workspace), _nbytes(workspace), _stream(stream)))


def topk_append(p, delta, workspace, stream=None):
    """Decode selection after one key is appended (p.N = the new cache length)."""
    check("dma_topk_append", load().dma_topk_append(ctypes.byref(p), _ptr(delta), _ptr(workspace),
                                                    _nbytes(workspace), _stream(stream)))


def gate_append(p, V, Delta, A, delta, x_save=None, stream=None):
    """Gate of the last key position only (delta[:, :, p.N - 1])."""
    check("dma_gate_append", load().dma_gate_append(ctypes.byref(p), _ptr(V), _ptr(Delta), _ptr(A), _ptr(delta),
                                                    _ptr(x_save), _stream(stream)))


def attn_fwd(p, Q, K, V, delta, evict, workspace, O, LSE, stream=None):
    check("dma_attn_fwd", load().dma_attn_fwd(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(delta),
                                              _ptr(evict), _ptr(workspace), _nbytes(workspace), _ptr(O),
                                              _ptr(LSE), _stream(stream)))


def attn_bwd(p, Q, K, V, delta, evict, workspace, O, LSE, dO, dQ, dK, dV, d_delta, stream=None):
    check("dma_attn_bwd", load().dma_attn_bwd(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(delta),
                                              _ptr(evict), _ptr(workspace), _nbytes(workspace), _ptr(O),
                                              _ptr(LSE), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV),
                                              _ptr(d_delta), _stream(stream)))


def gate_bwd(p, V, Delta, A, x_save, delta, d_delta, dDelta, dA, dV_gate, workspace, stream=None):
    check("dma_gate_bwd", load().dma_gate_bwd(ctypes.byref(p), _ptr(V), _ptr(Delta), _ptr(A),
                                              _ptr(x_save), _ptr(delta), _ptr(d_delta), _ptr(dDelta),
                                              _ptr(dA), _ptr(dV_gate), _ptr(workspace), _nbytes(workspace),
                                              _stream(stream)))


def gate_bwd_noalloc(p, V, Delta, A, x_save, delta, d_delta, dDelta, dA, dV_gate, stream=None):
    """dma_gate_bwd without a workspace, for callers that may not allocate device
    memory; its scratch is a fixed array inside the library (see include/dma.h)."""
    check("dma_gate_bwd_noalloc", load().dma_gate_bwd_noalloc(ctypes.byref(p), _ptr(V), _ptr(Delta), _ptr(A),
                                                              _ptr(x_save), _ptr(delta), _ptr(d_delta),
                                                              _ptr(dDelta), _ptr(dA), _ptr(dV_gate),
                                                              _stream(stream)))


def check_device_status(p, workspace, stream=None) -> int:
    code = ctypes.c_int32(0)
    load().dma_check_device_status(ctypes.byref(p), _ptr(workspace), _stream(stream), ctypes.byref(code))
    return int(code.value)


def selftest_bounded_wait(p, workspace, limit_cycles=1_000_000, stream=None):
    """Launch the device-side bounded-wait check (a wait that must give up and report)."""
    check("dma_selftest_bounded_wait", load().dma_selftest_bounded_wait(ctypes.byref(p), _ptr(workspace),
                                                                        _nbytes(workspace), int(limit_cycles),
                                                                        _stream(stream)))


def clear_device_status(p, workspace, stream=None):
    check("dma_clear_device_status", load().dma_clear_device_status(ctypes.byref(p), _ptr(workspace),
                                                                    _stream(stream)))


# ---------------------------------------------------------------- context-parallel prefill

def cp_layout(p, prefix_len, n_prev) -> DmaCpLayout:
    """Candidate-buffer and workspace sizes of shard problem p (see trainable_dynamic_mask_b200.cp)."""
    lay = DmaCpLayout()
    check("dma_cp_layout", load().dma_cp_layout(ctypes.byref(p), int(prefix_len), int(n_prev), ctypes.byref(lay)))
    return lay


def cp_candidates(p, shard_start, delta, K, V, cand, workspace, stream=None):
    check("dma_cp_candidates", load().dma_cp_candidates(ctypes.byref(p), int(shard_start), _ptr(delta), _ptr(K),
                                                        _ptr(V), _ptr(cand), _nbytes(cand), _ptr(workspace),
                                                        _nbytes(workspace), _stream(stream)))


def cp_compact(p, prefix_len, n_prev, cands, delta, K, V, delta_c, Kc, Vc, pos_c, workspace, stream=None):
    check("dma_cp_compact", load().dma_cp_compact(ctypes.byref(p), int(prefix_len), int(n_prev), _ptr(cands),
                                                  _nbytes(cands), _ptr(delta), _ptr(K), _ptr(V), _ptr(delta_c),
                                                  _ptr(Kc), _ptr(Vc), _ptr(pos_c), _ptr(workspace),
                                                  _nbytes(workspace), _stream(stream)))


# ---------------------------------------------------------------- convenience (torch allocation)

def alloc_workspace(p, device="cuda", stream=None):
    """A workspace for problem p (torch allocation) with its status word cleared."""
    import torch
    ws = torch.empty(workspace_size(p), dtype=torch.uint8, device=device)
    clear_device_status(p, ws, stream)
    return ws


def forward(p, Q, K, V, Delta, A, workspace=None, stream=None):
    """gate -> top-w mask -> attention forward.  Allocates the outputs (and the
    workspace if none is given) with torch on Q's device; returns a dict with
    delta, x, evict (None for decode), O, LSE, workspace."""
    import torch
    dev = Q.device
    ws = workspace if workspace is not None else alloc_workspace(p, dev, stream)
    f32 = torch.float32
    delta = torch.empty((p.B, p.H, p.N), dtype=f32, device=dev)
    x = torch.empty((p.B, p.H, p.N), dtype=f32, device=dev)
    decode = p.Nq == 1 and p.N > 1
    evict = None if decode else torch.empty((p.B, p.H, p.N), dtype=torch.int32, device=dev)
    O = torch.empty((p.B, p.H, p.Nq, p.d), dtype=Q.dtype, device=dev)
    LSE = torch.empty((p.B, p.H, p.Nq), dtype=f32, device=dev)
    gate(p, V, Delta, A, delta, x, ws, stream)
    topk_mask(p, delta, evict, ws, stream)
    attn_fwd(p, Q, K, V, delta, evict, ws, O, LSE, stream)
    return {"delta": delta, "x": x, "evict": evict, "O": O, "LSE": LSE, "workspace": ws}


def backward(p, Q, K, V, Delta, A, fwd, dO, stream=None):
    """Attention backward then gate backward for the outputs of forward().
    Returns dQ, dK, dV (attention part), dV_gate, d_delta, dDelta, dA."""
    import torch
    dev = Q.device
    f32 = torch.float32
    ws = fwd["workspace"]
    dQ = torch.empty_like(Q)
    dK = torch.empty_like(K)
    dV = torch.empty_like(V)
    dd = torch.empty((p.B, p.H, p.N), dtype=f32, device=dev)
    attn_bwd(p, Q, K, V, fwd["delta"], fwd["evict"], ws, fwd["O"], fwd["LSE"], dO, dQ, dK, dV, dd, stream)
    dDelta = torch.empty(tuple(Delta.shape), dtype=f32, device=dev)
    dA = torch.empty((p.H,), dtype=f32, device=dev)
    dVg = torch.empty(tuple(V.shape), dtype=f32, device=dev)
    gate_bwd(p, V, Delta, A, fwd["x"], fwd["delta"], dd, dDelta, dA, dVg, ws, stream)
    return {"dQ": dQ, "dK": dK, "dV": dV, "d_delta": dd, "dDelta": dDelta, "dA": dA, "dV_gate": dVg}
