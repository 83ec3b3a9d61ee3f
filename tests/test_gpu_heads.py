"""GPU parity with per-head windows ("adaptive window sizing", section "Future
Directions" of the page "Trainable Dynamic Mask Sparse Attention"; the window of
each head is supplied by the caller through dma_params_t.w_heads).

Against the oracle run head by head with that head's own window: eviction
indices, block lists and decode selections bit for bit; O, LSE and gradients
within |gpu - oracle| <= 2e-2 + 1e-2 |oracle|."""
import numpy as np
import pytest

import oracle
from workloads import get, make_delta, make_inputs

from gpu_common import assert_close, f32_dev, lib, to_dev, to_np, torch_cuda

pytestmark = pytest.mark.gpu


def _wh_dev(torch, w_heads):
    return torch.tensor(np.asarray(w_heads, dtype=np.int32), device="cuda")


def _check_lists(dma, p, ws, e_ref):
    B, H = p.B, p.H
    lay = dma.workspace_layout(p)
    wsn = ws.cpu().numpy()
    counts = wsn[lay.off_counts: lay.off_counts + B * H * lay.n_blocks * 8].view(np.int32).reshape(B, H, -1, 2)
    lists = wsn[lay.off_lists: lay.off_lists + B * H * lay.n_blocks * lay.list_cap * 4].view(np.int32).reshape(
        B, H, lay.n_blocks, lay.list_cap)
    for b in range(B):
        for h in range(H):
            for k, (full, part) in enumerate(oracle.live_keys_per_block(e_ref[b, h], 128)):
                nf, nl = counts[b, h, k]
                assert nf == full.size and nl == full.size + part.size, (b, h, k)
                np.testing.assert_array_equal(lists[b, h, k, :nf], full)
                np.testing.assert_array_equal(lists[b, h, k, nf:nl], part)


@pytest.mark.parametrize("N,w,w_heads,kind", [
    (300, 200, [1, 7, 128, 129, 200, 999], "uniform"),
    (1000, 512, [512, 64, 300, 0], "levels"),
    (4096, 2048, [2048, 1024, 256, 4096], "uniform"),
    (129, 64, [64, 1], "constant"),
])
def test_topk_mask_per_head_windows(N, w, w_heads, kind):
    dma = lib()
    torch = torch_cuda()
    B, H = 2, len(w_heads)
    d = make_delta((B, H, N), seed=N + w, kind=kind, levels=9)
    wh = _wh_dev(torch, w_heads)
    p = dma.make_params(B, H, H, N, 64, w, w_heads=wh)
    ws = dma.alloc_workspace(p)
    evict = torch.full((B, H, N), -7, dtype=torch.int32, device="cuda")
    dma.topk_mask(p, f32_dev(d), evict, ws)
    torch.cuda.synchronize()
    assert dma.check_device_status(p, ws) == 0
    e_ref = oracle.topw_eviction_heads(d, w_heads, w)
    np.testing.assert_array_equal(evict.cpu().numpy(), e_ref)
    _check_lists(dma, p, ws, e_ref)


ATTN_CASES = {
    "gqa_n700": (get("tiny").with_(B=2, H=4, Hkv=2, N=700, d=128, w=700, dtype="bf16", seed=81), [50, 300, 700, 129]),
    "mha_n333_d64": (get("tiny").with_(B=1, H=3, Hkv=3, N=333, d=64, w=100, dtype="bf16", seed=82), [1, 100, 37]),
    "prefill_heads": (get("prefill").with_(seed=83), [256, 512, 1024, 128] * 4),
}


@pytest.mark.parametrize("case", list(ATTN_CASES))
def test_attn_fwd_bwd_per_head_windows(case):
    wl, w_heads = ATTN_CASES[case]
    dma = lib()
    torch = torch_cuda()
    I = make_inputs(wl, with_dO=True)
    _, d64 = oracle.gate(I.V, I.Delta, I.A, gemm_dtype=np.float32 if wl.N > 1024 else np.float64)
    d32 = d64.astype(np.float32)
    wh = _wh_dev(torch, w_heads)
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, dtype=wl.dtype, w_heads=wh)
    ws = dma.alloc_workspace(p)
    Q, K, V, dO = (to_dev(getattr(I, n), I.bits.get(n), wl.dtype) for n in ("Q", "K", "V", "dO"))
    delta = f32_dev(d32)
    evict = torch.empty((wl.B, wl.H, wl.N), dtype=torch.int32, device="cuda")
    dma.topk_mask(p, delta, evict, ws)
    e_ref = oracle.topw_eviction_heads(d32, w_heads, wl.w)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(evict.cpu().numpy(), e_ref)
    O = torch.full_like(Q, float("nan"))
    LSE = torch.full((wl.B, wl.H, wl.N), float("nan"), dtype=torch.float32, device="cuda")
    dma.attn_fwd(p, Q, K, V, delta, evict, ws, O, LSE)
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    dd = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device="cuda")
    dma.attn_bwd(p, Q, K, V, delta, evict, ws, O, LSE, dO, dQ, dK, dV, dd)
    torch.cuda.synchronize()
    assert dma.check_device_status(p, ws) == 0
    gd = np.float32 if wl.N > 1024 else np.float64
    O_ref, L_ref = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e_ref, gemm_dtype=gd)
    assert_close(to_np(LSE), L_ref, "LSE")
    assert_close(to_np(O), O_ref, "O")
    r = oracle.attn_bwd(I.Q, I.K, I.V, d32.astype(np.float64), e_ref, I.dO, gemm_dtype=gd)
    for name, g, ref in zip(("dQ", "dK", "dV", "d_delta"), (dQ, dK, dV, dd), r):
        assert_close(to_np(g), ref, name)


def test_attn_fwd_chunk_per_head_windows():
    """A chunk of queries (the last 700 of 2500 positions) with per-head windows."""
    wl = get("tiny").with_(B=1, H=4, Hkv=2, N=2500, Nq=700, d=128, w=900, dtype="bf16", seed=84)
    w_heads = [900, 100, 513, 2]
    dma = lib()
    torch = torch_cuda()
    I = make_inputs(wl)
    _, d64 = oracle.gate(I.V, I.Delta, I.A, gemm_dtype=np.float32)
    d32 = d64.astype(np.float32)
    wh = _wh_dev(torch, w_heads)
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, Nq=wl.Nq, dtype="bf16", w_heads=wh)
    ws = dma.alloc_workspace(p)
    Q, K, V = (to_dev(getattr(I, n), I.bits.get(n), "bf16") for n in ("Q", "K", "V"))
    delta = f32_dev(d32)
    evict = torch.empty((wl.B, wl.H, wl.N), dtype=torch.int32, device="cuda")
    dma.topk_mask(p, delta, evict, ws)
    O = torch.full_like(Q, float("nan"))
    LSE = torch.full((wl.B, wl.H, wl.Nq), float("nan"), dtype=torch.float32, device="cuda")
    dma.attn_fwd(p, Q, K, V, delta, evict, ws, O, LSE)
    torch.cuda.synchronize()
    e_ref = oracle.topw_eviction_heads(d32, w_heads, wl.w)
    np.testing.assert_array_equal(evict.cpu().numpy(), e_ref)
    O_ref, L_ref = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e_ref, q_pos0=wl.N - wl.Nq,
                                   gemm_dtype=np.float32)
    assert_close(to_np(LSE), L_ref, "LSE")
    assert_close(to_np(O), O_ref, "O")


def _sel_rows(dma, p, ws, w_heads):
    lay = dma.workspace_layout(p)
    sel = ws.cpu().numpy()[lay.off_sel: lay.off_sel + p.B * p.H * lay.sel_len * 4].view(np.int32)
    sel = sel.reshape(p.B * p.H, lay.sel_len)
    W = oracle.head_windows(w_heads, p.w)
    return [sel[r, :min(p.N, int(W[r % p.H]))] for r in range(p.B * p.H)]


def test_decode_per_head_windows():
    wl = get("decode").with_(B=2, H=4, Hkv=2, N=5000, w=1000, seed=85)
    w_heads = [1000, 10, 257, 600]
    dma = lib()
    torch = torch_cuda()
    I = make_inputs(wl)
    _, d64 = oracle.gate(I.V, I.Delta, I.A, gemm_dtype=np.float32)
    d32 = d64.astype(np.float32)
    wh = _wh_dev(torch, w_heads)
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, Nq=1, dtype="bf16", w_heads=wh)
    assert dma.workspace_layout(p).sel_len == wl.w
    ws = dma.alloc_workspace(p)
    delta = f32_dev(d32)
    dma.topk_mask(p, delta, None, ws)
    Q, K, V = (to_dev(getattr(I, n), I.bits.get(n), "bf16") for n in ("Q", "K", "V"))
    O = torch.full((wl.B, wl.H, 1, wl.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    LSE = torch.full((wl.B, wl.H, 1), float("nan"), dtype=torch.float32, device="cuda")
    dma.attn_fwd(p, Q, K, V, delta, None, ws, O, LSE)
    torch.cuda.synchronize()
    got = _sel_rows(dma, p, ws, w_heads)
    ref = oracle.decode_select_heads(d32, w_heads, wl.w)
    for r in range(wl.B * wl.H):
        np.testing.assert_array_equal(got[r], ref[r], err_msg=f"row {r}")
    o_ref = np.empty((wl.B, wl.H, wl.d))
    l_ref = np.empty((wl.B, wl.H))
    for b in range(wl.B):
        for h in range(wl.H):
            o1, l1 = oracle.decode_attn(I.Q[b:b + 1, h:h + 1], I.K[b:b + 1, h // wl.G: h // wl.G + 1],
                                        I.V[b:b + 1, h // wl.G: h // wl.G + 1], d32[b:b + 1, h:h + 1].astype(np.float64),
                                        ref[b * wl.H + h][None, None])
            o_ref[b, h], l_ref[b, h] = o1[0, 0], l1[0, 0]
    assert_close(to_np(LSE)[:, :, 0], l_ref, "LSE")
    assert_close(to_np(O)[:, :, 0], o_ref, "O")


def test_decode_append_per_head_windows():
    """Keys appended one by one from an empty cache past every head's window: after each, every
    row equals the oracle's selection over the prefix with that row's window."""
    dma = lib()
    torch = torch_cuda()
    B, H, L, w = 2, 3, 90, 40
    w_heads = [40, 5, 17]
    d = make_delta((B, H, L), seed=86, kind="levels", levels=7)
    wh = _wh_dev(torch, w_heads)
    ws = dma.alloc_workspace(dma.make_params(B, H, H, L, 128, w, Nq=1, w_heads=wh))
    for n in range(2, L + 1):
        p = dma.make_params(B, H, H, n, 128, w, Nq=1, w_heads=wh)
        dma.topk_append(p, f32_dev(d[:, :, :n]), ws)
        torch.cuda.synchronize()
        got = _sel_rows(dma, p, ws, w_heads)
        ref = oracle.decode_select_heads(d[:, :, :n], w_heads, w)
        for r in range(B * H):
            np.testing.assert_array_equal(got[r], ref[r], err_msg=f"L={n} row {r}")
