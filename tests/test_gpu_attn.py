"""GPU parity of masked attention forward, backward, gate backward and decode,
called through the C ABI, against the CPU oracle on the same seeded inputs.

Tolerance: |gpu - oracle| <= 2e-2 + 1e-2 |oracle| for O, LSE and every
gradient.  The selection fed to both sides comes from the oracle's delta
(float32), and the GPU's own eviction indices are checked bit-exact first."""
import numpy as np
import pytest

import oracle
from workloads import get, make_inputs

from gpu_common import assert_close, f32_dev, lib, to_dev, to_np, torch_cuda

pytestmark = pytest.mark.gpu


def _setup(wl, with_dO=False, bf16_values=False):
    """Inputs on both sides, the oracle's delta and eviction index, and the
    GPU mask built from that delta."""
    dma = lib()
    torch = torch_cuda()
    I = make_inputs(wl, with_dO=with_dO, bf16_values=bf16_values)
    big = wl.N * wl.B > 4096
    _, d64 = oracle.gate(I.V, I.Delta, I.A, gemm_dtype=np.float32 if big else np.float64)
    d32 = d64.astype(np.float32)
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, Nq=wl.Nq, dtype=wl.dtype)
    ws = torch.empty(dma.workspace_size(p), dtype=torch.uint8, device="cuda")
    dev = {
        "Q": to_dev(I.Q, I.bits.get("Q"), wl.dtype),
        "K": to_dev(I.K, I.bits.get("K"), wl.dtype),
        "V": to_dev(I.V, I.bits.get("V"), wl.dtype),
        "delta": f32_dev(d32),
    }
    if with_dO:
        dev["dO"] = to_dev(I.dO, I.bits.get("dO"), wl.dtype)
    e_ref = None
    if not (wl.Nq == 1 and wl.N > 1):   # prefill, training or a chunk of queries: eviction indices
        e_ref = np.stack([np.stack([oracle.topw_eviction(d32[b, h], wl.w) for h in range(wl.H)])
                          for b in range(wl.B)])
        dev["evict"] = torch.empty((wl.B, wl.H, wl.N), dtype=torch.int32, device="cuda")
        dma.topk_mask(p, dev["delta"], dev["evict"], ws)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(dev["evict"].cpu().numpy(), e_ref)
    else:
        dev["evict"] = None
        dma.topk_mask(p, dev["delta"], None, ws)
    return dma, torch, I, p, ws, dev, d32, e_ref


def _fwd(dma, torch, wl, p, ws, dev):
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    O = torch.full((wl.B, wl.H, wl.Nq, wl.d), float("nan"), dtype=dt, device="cuda")
    LSE = torch.full((wl.B, wl.H, wl.Nq), float("nan"), dtype=torch.float32, device="cuda")
    dma.attn_fwd(p, dev["Q"], dev["K"], dev["V"], dev["delta"], dev["evict"], ws, O, LSE)
    torch.cuda.synchronize()
    return O, LSE


FWD_CASES = {
    "tiny": get("tiny"),
    "prefill": get("prefill"),
    "odd_n129_w7_d64": get("tiny").with_(B=2, H=4, Hkv=2, N=129, d=64, w=7, dtype="bf16", seed=21),
    "n1": get("tiny").with_(B=1, H=2, Hkv=2, N=1, d=128, w=1, dtype="bf16", seed=22),
    "n300_w_ge_n": get("tiny").with_(B=1, H=2, Hkv=1, N=300, d=128, w=400, dtype="bf16", seed=23),
    "n300_w1": get("tiny").with_(B=1, H=2, Hkv=1, N=300, d=128, w=1, dtype="f32", seed=24),
    "mha_n1000_w200": get("tiny").with_(B=2, H=3, Hkv=3, N=1000, d=128, w=200, dtype="bf16", seed=25),
}


CHUNK_CASES = {   # the queries are the last Nq positions of the N keys (chunked prefill)
    "n3000_q700_w500": get("tiny").with_(B=1, H=4, Hkv=2, N=3000, Nq=700, d=128, w=500, dtype="bf16", seed=61),
    "n4096_q1000_w1024": get("prefill").with_(H=4, Hkv=2, N=4096, Nq=1000, seed=62),
    "n2048_q256_w300_d64": get("tiny").with_(B=2, H=2, Hkv=1, N=2048, Nq=256, d=64, w=300, dtype="bf16", seed=63),
    "n1500_q1499_w200": get("tiny").with_(B=1, H=2, Hkv=2, N=1500, Nq=1499, d=128, w=200, dtype="bf16", seed=64),
    "n700_q3_w_ge_n": get("tiny").with_(B=1, H=2, Hkv=1, N=700, Nq=3, d=128, w=900, dtype="f32", seed=65),
}


@pytest.mark.parametrize("case", list(CHUNK_CASES))
def test_attn_fwd_chunked(case):
    wl = CHUNK_CASES[case]
    dma, torch, I, p, ws, dev, d32, e_ref = _setup(wl)
    O, LSE = _fwd(dma, torch, wl, p, ws, dev)
    O_ref, L_ref = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e_ref, q_pos0=wl.N - wl.Nq,
                                   gemm_dtype=np.float32 if wl.N > 1024 else np.float64)
    assert_close(to_np(LSE), L_ref, "LSE")
    assert_close(to_np(O), O_ref, "O")


@pytest.mark.parametrize("case", list(FWD_CASES))
def test_attn_fwd_full(case):
    wl = FWD_CASES[case]
    dma, torch, I, p, ws, dev, d32, e_ref = _setup(wl)
    O, LSE = _fwd(dma, torch, wl, p, ws, dev)
    O_ref, L_ref = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e_ref,
                                   gemm_dtype=np.float32 if wl.N > 1024 else np.float64)
    assert_close(to_np(LSE), L_ref, "LSE")
    assert_close(to_np(O), O_ref, "O")


def test_attn_fwd_forward_only_flag_same_outputs():
    """DMA_FLAG_FORWARD_ONLY changes what the forward keeps for a backward, never its outputs:
    O and LSE bit for bit equal to those of the same problem without the flag (a shape whose pairs
    are not split, so that no merge order can differ between the two runs)."""
    wl = get("prefill").with_(H=32, Hkv=8, seed=27)
    dma, torch, I, p, ws, dev, d32, e_ref = _setup(wl)
    O, LSE = _fwd(dma, torch, wl, p, ws, dev)
    p1 = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, dtype=wl.dtype, forward_only=True)
    ws1 = dma.alloc_workspace(p1)
    dma.topk_mask(p1, dev["delta"], dev["evict"], ws1)
    O1, LSE1 = _fwd(dma, torch, wl, p1, ws1, dev)
    assert torch.equal(O.view(torch.int16), O1.view(torch.int16)) and torch.equal(LSE, LSE1)
    rows = _sample_rows(wl.N, 512, 98)
    O_ref, L_ref = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e_ref, rows=rows, gemm_dtype=np.float32)
    assert_close(to_np(O1)[:, :, rows], O_ref[:, :, rows], "O")


def _sample_rows(N, n, seed):
    """A seeded sample of n query rows that always holds both edges of every pair
    of 128-row blocks near the start and the end (row 0, the first block edges,
    the last full pair and the ragged tail)."""
    rng = np.random.default_rng(seed)
    edges = np.array([0, 1, 127, 128, 255, 256, N - 257, N - 256, N - 129, N - 128, N - 1])
    edges = edges[(edges >= 0) & (edges < N)]
    rest = rng.choice(np.setdiff1d(np.arange(N), edges), size=max(0, n - edges.size), replace=False)
    return np.unique(np.concatenate([edges, rest]))


def test_attn_fwd_long_sampled_rows_full_size():
    """The long workload at full size in the benchmark's launch configuration;
    the oracle recomputes a seeded sample of 2048 query rows of every head (the
    same rows in every head; block edges and the ragged end included).  The
    training workload's forward is checked in full with its backward below."""
    wl = get("long")
    dma, torch, I, p, ws, dev, d32, e_ref = _setup(wl)
    O, LSE = _fwd(dma, torch, wl, p, ws, dev)
    rows = _sample_rows(wl.N, 2048, 99)
    assert rows.size == 2048
    O_ref, L_ref = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e_ref, rows=rows, gemm_dtype=np.float32)
    assert_close(to_np(LSE)[:, :, rows], L_ref[:, :, rows], "LSE")
    assert_close(to_np(O)[:, :, rows], O_ref[:, :, rows], "O")


# ---------------------------------------------------------------- backward

BWD_CASES = {
    "tiny": get("tiny"),
    "odd_n200_w13": get("tiny").with_(B=2, H=4, Hkv=2, N=200, d=128, w=13, dtype="bf16", seed=31),
    "n1": get("tiny").with_(B=1, H=1, Hkv=1, N=1, d=64, w=1, dtype="bf16", seed=32),
    "gqa_n700_w300": get("tiny").with_(B=1, H=8, Hkv=2, N=700, d=128, w=300, dtype="bf16", seed=33),
    "w_ge_n_d64": get("tiny").with_(B=1, H=2, Hkv=1, N=333, d=64, w=512, dtype="bf16", seed=34),
}


def _bwd(dma, torch, wl, p, ws, dev, O, LSE):
    dQ = torch.empty_like(dev["Q"])
    dK = torch.empty_like(dev["K"])
    dV = torch.empty_like(dev["V"])
    dd = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device="cuda")
    dma.attn_bwd(p, dev["Q"], dev["K"], dev["V"], dev["delta"], dev["evict"], ws, O, LSE, dev["dO"], dQ, dK, dV, dd)
    torch.cuda.synchronize()
    return dQ, dK, dV, dd


@pytest.mark.parametrize("case", list(BWD_CASES))
def test_attn_bwd_full(case):
    """For float32 storage the attention kernels round Q, K, V and dO to bf16
    when they load them; the backward check feeds bf16-representable float32
    values so that it measures the kernels' arithmetic against the tolerance
    (the float32 forward is checked on unrounded values above)."""
    wl = BWD_CASES[case]
    dma, torch, I, p, ws, dev, d32, e_ref = _setup(wl, with_dO=True, bf16_values=True)
    O, LSE = _fwd(dma, torch, wl, p, ws, dev)
    dQ, dK, dV, dd = _bwd(dma, torch, wl, p, ws, dev, O, LSE)
    r = oracle.attn_bwd(I.Q, I.K, I.V, d32.astype(np.float64), e_ref, I.dO)
    for name, g, ref in zip(("dQ", "dK", "dV", "d_delta"), (dQ, dK, dV, dd), r):
        assert_close(to_np(g), ref, name)


def test_attn_bwd_train_full_size_every_head():
    """The training workload at full size on the GPU (the benchmark's launch
    configuration): O and LSE of every query row, then every gradient of every
    head, batch row and KV group against the oracle's dense analytic backward
    (float32 GEMMs, float64 row reductions), element by element: dQ, dK, dV and
    d_delta in full."""
    wl = get("train")
    dma, torch, I, p, ws, dev, d32, e_ref = _setup(wl, with_dO=True)
    O, LSE = _fwd(dma, torch, wl, p, ws, dev)
    dQ, dK, dV, dd = _bwd(dma, torch, wl, p, ws, dev, O, LSE)
    got = [to_np(t) for t in (dQ, dK, dV, dd)]
    del dQ, dK, dV, dd
    O_ref, L_ref = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e_ref, gemm_dtype=np.float32)
    assert_close(to_np(LSE), L_ref, "LSE")
    assert_close(to_np(O), O_ref, "O")
    del O_ref, L_ref
    r = oracle.attn_bwd(I.Q, I.K, I.V, d32.astype(np.float64), e_ref, I.dO, gemm_dtype=np.float32)
    for name, g, ref in zip(("dQ", "dK", "dV", "d_delta"), got, r):
        assert_close(g, ref, name)


# ---------------------------------------------------------------- gate backward

@pytest.mark.parametrize("wl", [get("tiny"), get("prefill"),
                                get("tiny").with_(B=2, H=6, Hkv=3, N=333, d=64, dtype="bf16", seed=41)],
                         ids=["tiny", "prefill", "odd"])
def test_gate_bwd(wl):
    dma = lib()
    torch = torch_cuda()
    I = make_inputs(wl)
    rng = np.random.default_rng(wl.seed + 1000)
    g = rng.standard_normal((wl.B, wl.H, wl.N)).astype(np.float32)
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, dtype=wl.dtype)
    ws = torch.empty(dma.workspace_size(p), dtype=torch.uint8, device="cuda")
    V = to_dev(I.V, I.bits.get("V"), wl.dtype)
    D = to_dev(I.Delta, I.bits.get("Delta"), wl.dtype)
    A = f32_dev(I.A)
    delta = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device="cuda")
    x = torch.empty_like(delta)
    dma.gate(p, V, D, A, delta, x)
    dDelta = torch.empty((wl.Hkv * wl.d, wl.H), dtype=torch.float32, device="cuda")
    dA = torch.empty((wl.H,), dtype=torch.float32, device="cuda")
    dVg = torch.empty((wl.B, wl.Hkv, wl.N, wl.d), dtype=torch.float32, device="cuda")
    dma.gate_bwd(p, V, D, A, x, delta, f32_dev(g), dDelta, dA, dVg, ws)
    torch.cuda.synchronize()
    rD, rA, rV = oracle.gate_bwd(I.V, I.Delta, I.A, g.astype(np.float64))
    assert_close(to_np(dDelta), rD, "dDelta")
    assert_close(to_np(dA), rA, "dA")
    assert_close(to_np(dVg), rV, "dV_gate")


# ---------------------------------------------------------------- decode

DECODE_CASES = {
    "small": get("decode").with_(B=2, N=5000, w=300, seed=51),
    "w_ge_L": get("decode").with_(B=1, H=4, Hkv=2, N=1000, w=4096, seed=52),
    "d64_f32": get("decode").with_(B=1, H=2, Hkv=1, N=3000, d=64, w=700, dtype="f32", seed=53),
    "full": get("decode"),
}


@pytest.mark.parametrize("case", list(DECODE_CASES))
def test_decode(case):
    wl = DECODE_CASES[case]
    dma, torch, I, p, ws, dev, d32, _ = _setup(wl)
    lay = dma.workspace_layout(p)
    sel = ws.cpu().numpy()[lay.off_sel: lay.off_sel + wl.B * wl.H * lay.sel_len * 4].view(np.int32)
    sel = sel.reshape(wl.B, wl.H, lay.sel_len)
    sel_ref = oracle.decode_select(d32, wl.w)
    np.testing.assert_array_equal(sel, sel_ref)
    O, LSE = _fwd(dma, torch, wl, p, ws, dev)
    o_ref, l_ref = oracle.decode_attn(I.Q, I.K, I.V, d32.astype(np.float64), sel_ref)
    assert_close(to_np(LSE)[:, :, 0], l_ref, "LSE")
    assert_close(to_np(O)[:, :, 0], o_ref, "O")


# ---------------------------------------------------------------- public chain

def test_forward_backward_chain_on_tiny():
    """dma.forward / dma.backward (gate -> mask -> attention -> backward ->
    gate backward) on the tiny workload, each output against the oracle."""
    dma = lib()
    torch = torch_cuda()
    wl = get("tiny")
    I = make_inputs(wl, with_dO=True, bf16_values=True)   # see test_attn_bwd_full
    p = dma.make_params(wl.B, wl.H, wl.Hkv, wl.N, wl.d, wl.w, dtype=wl.dtype)
    Q, K, V = f32_dev(I.Q), f32_dev(I.K), f32_dev(I.V)
    Dl, A, dO = f32_dev(I.Delta), f32_dev(I.A), f32_dev(I.dO)
    fwd = dma.forward(p, Q, K, V, Dl, A)
    bwd = dma.backward(p, Q, K, V, Dl, A, fwd, dO)
    torch.cuda.synchronize()
    _, d64 = oracle.gate(I.V, I.Delta, I.A)
    d_gpu = to_np(fwd["delta"])
    np.testing.assert_allclose(d_gpu, d64, rtol=1e-5)
    # the oracle's selection on the GPU's delta (a near-tie could flip otherwise) must equal the GPU's
    e_ref = np.stack([np.stack([oracle.topw_eviction(d_gpu[0, h].astype(np.float32), wl.w) for h in range(wl.H)])])
    np.testing.assert_array_equal(fwd["evict"].cpu().numpy(), e_ref)
    O_ref, L_ref = oracle.attn_fwd(I.Q, I.K, I.V, d64, e_ref)
    assert_close(to_np(fwd["O"]), O_ref, "O")
    assert_close(to_np(fwd["LSE"]), L_ref, "LSE")
    dQ, dK, dV, dd = oracle.attn_bwd(I.Q, I.K, I.V, d64, e_ref, I.dO)
    assert_close(to_np(bwd["dQ"]), dQ, "dQ")
    assert_close(to_np(bwd["dK"]), dK, "dK")
    assert_close(to_np(bwd["dV"]), dV, "dV")
    assert_close(to_np(bwd["d_delta"]), dd, "d_delta")
    rD, rA, rV = oracle.gate_bwd(I.V, I.Delta, I.A, dd)
    assert_close(to_np(bwd["dDelta"]), rD, "dDelta")
    assert_close(to_np(bwd["dA"]), rA, "dA")
    assert_close(to_np(bwd["dV_gate"]), rV, "dV_gate")
