"""GPU parity of the gate (delta) and of the causal top-w mask encoding,
called through the C ABI, against the CPU oracle.

delta within 1e-5 relative; eviction indices, block lists and counts bit for
bit given the same delta (the oracle's delta, rounded to float32, is the input
of both sides)."""
import numpy as np
import pytest

import oracle
from workloads import get, make_delta, make_inputs

from gpu_common import assert_delta_close, f32_dev, lib, to_dev, to_np, torch_cuda

pytestmark = pytest.mark.gpu


def _gate_case(wl):
    dma = lib()
    torch = torch_cuda()
    I = make_inputs(wl)
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, Nq=wl.Nq, dtype=wl.dtype)
    V = to_dev(I.V, I.bits.get("V"), wl.dtype)
    D = to_dev(I.Delta, I.bits.get("Delta"), wl.dtype)
    A = f32_dev(I.A)
    delta = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device="cuda")
    x = torch.empty_like(delta)
    dma.gate(p, V, D, A, delta, x)
    torch.cuda.synchronize()
    x_ref, d_ref = oracle.gate(I.V, I.Delta, I.A, gemm_dtype=np.float64 if wl.N * wl.B <= 65536 else np.float32)
    assert_delta_close(to_np(delta), d_ref)
    np.testing.assert_allclose(to_np(x), x_ref, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("name", ["tiny", "prefill", "long", "train"])
def test_gate_workloads(name):
    _gate_case(get(name))


@pytest.mark.parametrize("shape", [
    dict(B=1, H=1, Hkv=1, N=1, d=64, w=1),
    dict(B=2, H=3, Hkv=1, N=7, d=64, w=2),
    dict(B=1, H=6, Hkv=2, N=130, d=128, w=9),
    dict(B=3, H=32, Hkv=8, N=65, d=128, w=16),
])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gate_odd_shapes(shape, dtype):
    _gate_case(get("tiny").with_(dtype=dtype, seed=11, **shape))


# ---------------------------------------------------------------- top-w

def _topw_case(B, H, N, w, delta_np):
    dma = lib()
    torch = torch_cuda()
    p = dma.make_params(B, H, H, N, 64, w)
    ws = torch.empty(dma.workspace_size(p), dtype=torch.uint8, device="cuda")
    dma.clear_device_status(p, ws)
    delta = f32_dev(delta_np)
    evict = torch.full((B, H, N), -7, dtype=torch.int32, device="cuda")
    dma.topk_mask(p, delta, evict, ws)
    torch.cuda.synchronize()
    assert dma.check_device_status(p, ws) == 0
    lay = dma.workspace_layout(p)
    e_gpu = evict.cpu().numpy()
    wsn = ws.cpu().numpy()
    counts = wsn[lay.off_counts: lay.off_counts + B * H * lay.n_blocks * 8].view(np.int32).reshape(B, H, lay.n_blocks, 2)
    lists = wsn[lay.off_lists: lay.off_lists + B * H * lay.n_blocks * lay.list_cap * 4].view(np.int32).reshape(
        B, H, lay.n_blocks, lay.list_cap)
    for b in range(B):
        for h in range(H):
            e_ref = oracle.topw_eviction(delta_np[b, h], w)
            if not np.array_equal(e_gpu[b, h], e_ref):
                bad = np.nonzero(e_gpu[b, h] != e_ref)[0]
                raise AssertionError(f"evict mismatch at (b={b},h={h}) keys {bad[:8]}: gpu {e_gpu[b, h][bad[:8]]} "
                                     f"oracle {e_ref[bad[:8]]}")
            for k, (full, part) in enumerate(oracle.live_keys_per_block(e_ref, 128)):
                nf, nl = counts[b, h, k]
                assert nf == full.size and nl == full.size + part.size, (b, h, k)
                np.testing.assert_array_equal(lists[b, h, k, :nf], full)
                np.testing.assert_array_equal(lists[b, h, k, nf:nl], part)


@pytest.mark.parametrize("name", ["tiny", "prefill", "train", "long"])
def test_topw_on_oracle_delta(name):
    wl = get(name)
    I = make_inputs(wl)
    _, d = oracle.gate(I.V, I.Delta, I.A, gemm_dtype=np.float32 if wl.N > 1024 else np.float64)
    _topw_case(wl.B, wl.H, wl.N, wl.w, d.astype(np.float32))


@pytest.mark.parametrize("kind,levels", [("uniform", 0), ("levels", 3), ("levels", 50), ("increasing", 0),
                                         ("decreasing", 0), ("constant", 0)])
@pytest.mark.parametrize("N,w", [(1, 1), (5, 2), (127, 1), (128, 128), (129, 64), (300, 7), (300, 299),
                                 (300, 300), (300, 1000), (1000, 200), (2049, 512)])
def test_topw_synthetic(kind, levels, N, w):
    d = make_delta((2, 2, N), seed=N * 7 + w, kind=kind, levels=levels)
    _topw_case(2, 2, N, w, d)


def test_topw_max_row_with_ties():
    """Largest supported row (16384) with heavy ties: exercises every radix
    pass and the tie rule at full size."""
    d = make_delta((1, 2, 16384), seed=5, kind="levels", levels=97)
    _topw_case(1, 2, 16384, 2048, d)


def test_topw_negative_and_zero_values():
    """The order covers any non-NaN float: negative values, -0.0 == +0.0."""
    rng = np.random.default_rng(3)
    d = rng.standard_normal((1, 2, 700)).astype(np.float32)
    d[0, 0, ::5] = 0.0
    d[0, 0, 1::5] = -0.0
    d[0, 1, :50] = -np.inf
    _topw_case(1, 2, 700, 33, d)


# ---------------------------------------------------------------- decode selection

@pytest.mark.parametrize("L,w,kind", [(1000, 64, "uniform"), (4096, 2048, "levels"), (5000, 5000, "uniform"),
                                      (777, 3, "constant"), (65536, 2048, "uniform")])
def test_decode_select(L, w, kind):
    dma = lib()
    torch = torch_cuda()
    B, H = 2, 2
    d = make_delta((B, H, L), seed=L + w, kind=kind, levels=20)
    p = dma.make_params(B, H, H, L, 128, w, Nq=1)
    ws = torch.empty(dma.workspace_size(p), dtype=torch.uint8, device="cuda")
    dma.topk_mask(p, f32_dev(d), None, ws)
    torch.cuda.synchronize()
    lay = dma.workspace_layout(p)
    sel = ws.cpu().numpy()[lay.off_sel: lay.off_sel + B * H * lay.sel_len * 4].view(np.int32).reshape(B, H, -1)
    np.testing.assert_array_equal(sel, oracle.decode_select(d, w))


# ---------------------------------------------------------------- decode: one key appended

def _sel_of(dma, p, ws):
    lay = dma.workspace_layout(p)
    B, H = p.B, p.H
    return ws.cpu().numpy()[lay.off_sel: lay.off_sel + B * H * lay.sel_len * 4].view(np.int32).reshape(B, H, -1)


@pytest.mark.parametrize("L0,L,w,kind", [(2, 70, 16, "uniform"), (2, 70, 16, "levels"), (30, 200, 33, "constant"),
                                         (3000, 3012, 2048, "levels"), (65535, 65536, 2048, "uniform")])
def test_decode_select_append(L0, L, w, kind):
    """dma_topk_append grows the selection key by key (from none while L <= w + 1, else from
    dma_topk_mask at L0); after every key it equals the oracle's selection over the whole prefix."""
    dma = lib()
    torch = torch_cuda()
    B, H = 2, 3
    d = make_delta((B, H, L), seed=L0 + L + w, kind=kind, levels=6)
    ws = torch.empty(dma.workspace_size(dma.make_params(B, H, H, L, 128, w, Nq=1)), dtype=torch.uint8, device="cuda")
    if L0 - 1 > w:
        p0 = dma.make_params(B, H, H, L0 - 1, 128, w, Nq=1)
        dma.topk_mask(p0, f32_dev(d[:, :, :L0 - 1]), None, ws)
    for n in range(L0, L + 1):
        p = dma.make_params(B, H, H, n, 128, w, Nq=1)
        dma.topk_append(p, f32_dev(d[:, :, :n]), ws)
        torch.cuda.synchronize()
        if n == L or n - L0 < 40 or n % 17 == 0:
            np.testing.assert_array_equal(_sel_of(dma, p, ws), oracle.decode_select(d[:, :, :n], w), err_msg=f"L={n}")
    # the decode attention reads delta from the copy the appends kept beside the selection
    rng = np.random.default_rng(L + w)
    bf = lambda a: torch.from_numpy(a).to("cuda").bfloat16()
    q, Kc, Vc = (bf(rng.standard_normal(s).astype(np.float32)) for s in ((B, H, 1, 128), (B, H, L, 128), (B, H, L, 128)))
    O = torch.empty((B, H, 1, 128), dtype=torch.bfloat16, device="cuda")
    LSE = torch.empty((B, H, 1), dtype=torch.float32, device="cuda")
    dma.attn_fwd(p, q, Kc, Vc, f32_dev(d), None, ws, O, LSE)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.decode_attn(to_np(q), to_np(Kc), to_np(Vc), d.astype(np.float64), oracle.decode_select(d, w))
    np.testing.assert_allclose(to_np(LSE)[:, :, 0], l_ref, atol=2e-2, rtol=1e-2)
    np.testing.assert_allclose(to_np(O)[:, :, 0], o_ref, atol=2e-2, rtol=1e-2)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gate_append(dtype):
    """dma_gate_append writes delta (and x) at position N-1 only, within the gate's tolerance."""
    dma = lib()
    torch = torch_cuda()
    wl = get("decode").with_(B=2, N=3000, dtype=dtype, seed=71)
    I = make_inputs(wl)
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, Nq=1, dtype=dtype)
    V = to_dev(I.V, I.bits.get("V"), dtype)
    D = to_dev(I.Delta, I.bits.get("Delta"), dtype)
    delta = torch.full((wl.B, wl.H, wl.N), float("nan"), dtype=torch.float32, device="cuda")
    x = torch.full_like(delta, float("nan"))
    dma.gate_append(p, V, D, f32_dev(I.A), delta, x)
    torch.cuda.synchronize()
    x_ref, d_ref = oracle.gate(I.V, I.Delta, I.A)
    got_d, got_x = to_np(delta), to_np(x)
    assert_delta_close(got_d[:, :, -1:], d_ref[:, :, -1:])
    np.testing.assert_allclose(got_x[:, :, -1], x_ref[:, :, -1], rtol=1e-5, atol=1e-5)
    assert np.isnan(got_d[:, :, :-1]).all() and np.isnan(got_x[:, :, :-1]).all()
