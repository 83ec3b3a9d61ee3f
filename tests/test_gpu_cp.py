"""Context-parallel prefill on the GPU, the ranks emulated one after another on a
single GPU (no rank waits on another: the exchange is a host-side stack of the
candidate buffers, the collective itself is covered by the gloo test).

Per shard, through the C ABI: the candidate buffer equals the oracle's
candidates bit for bit; the compacted sequence (rows, delta, positions) equals
the oracle's compaction bit for bit; its selection equals the oracle's
selection on the same compacted delta; the shard's O and LSE equal the rows of
the whole sequence's oracle attention within |gpu - oracle| <= 2e-2 + 1e-2 |oracle|."""
import numpy as np
import pytest

import oracle
from workloads import get, make_inputs

from gpu_common import assert_close, f32_dev, lib, to_dev, to_np, torch_cuda

pytestmark = pytest.mark.gpu


def _cand_arrays(dma, p, cand, B, H, w, d):
    lay = dma.cp_layout(p, 0, 0)
    c = cand.cpu().numpy()
    pos = c[lay.off_pos: lay.off_pos + B * H * w * 4].view(np.int32).reshape(B, H, w)
    dl = c[lay.off_delta: lay.off_delta + B * H * w * 4].view(np.float32).reshape(B, H, w)
    K = c[lay.off_k: lay.off_k + B * H * w * d * 2].view(np.uint16).reshape(B, H, w, d)
    V = c[lay.off_v: lay.off_v + B * H * w * d * 2].view(np.uint16).reshape(B, H, w, d)
    return pos, dl, K, V


CASES = {
    "r2_w200": (get("tiny").with_(B=2, H=4, Hkv=2, N=1500, d=128, w=200, dtype="bf16", seed=91), 2, None),
    "r3_ragged_d64": (get("tiny").with_(B=1, H=4, Hkv=1, N=1000, d=64, w=150, dtype="bf16", seed=92), 3, None),
    "r4_heads": (get("tiny").with_(B=1, H=4, Hkv=2, N=2048, d=128, w=300, dtype="bf16", seed=93), 4,
                 [300, 17, 128, 256]),
    "r2_w_above_shard": (get("tiny").with_(B=1, H=2, Hkv=1, N=600, d=128, w=512, dtype="bf16", seed=94), 2, None),
    "long_r2": (get("long"), 2, None),
}


@pytest.mark.parametrize("case", list(CASES))
def test_cp_shards_equal_whole_sequence(case):
    from trainable_dynamic_mask_b200 import cp
    wl, R, w_heads = CASES[case]
    dma = lib()
    torch = torch_cuda()
    I = make_inputs(wl)
    big = wl.N * wl.H > 100000
    _, d64 = oracle.gate(I.V, I.Delta, I.A, gemm_dtype=np.float32 if big else np.float64)
    d32 = d64.astype(np.float32)
    wh = None if w_heads is None else torch.tensor(np.asarray(w_heads, np.int32), device="cuda")
    bounds = cp.shard_bounds(wl.N, R)
    e_full = oracle.topw_eviction_heads(d32, np.full(wl.H, wl.w) if w_heads is None else w_heads, wl.w)
    Q, K, V = (to_dev(getattr(I, n), I.bits.get(n), "bf16") for n in ("Q", "K", "V"))
    delta = f32_dev(d32)
    # every rank's candidates (the exchange: a stack of the buffers)
    cands, ps = [], []
    for r, (s0, s1) in enumerate(bounds):
        p = dma.make_params(wl.B, wl.H, wl.Hkv, s1 - s0, wl.d, wl.w, dtype="bf16", w_heads=wh)
        ps.append(p)
        cand = cp.candidates(p, s0, delta[:, :, s0:s1].contiguous(), K[:, :, s0:s1].contiguous(),
                             V[:, :, s0:s1].contiguous())
        torch.cuda.synchronize()
        ref = oracle.cp_candidates(d32[:, :, s0:s1], I.K[:, :, s0:s1], I.V[:, :, s0:s1], w_heads, wl.w, s0)
        pos, dl, Kb, Vb = _cand_arrays(dma, p, cand, wl.B, wl.H, wl.w, wl.d)
        np.testing.assert_array_equal(pos, ref["pos"])
        np.testing.assert_array_equal(dl, ref["delta"])
        np.testing.assert_array_equal(Kb, _bits_rows(I, "K", ref, wl))
        np.testing.assert_array_equal(Vb, _bits_rows(I, "V", ref, wl))
        cands.append((cand, ref))
    allc = torch.stack([c for c, _ in cands])
    rows = np.arange(wl.N) if not big else np.unique(np.concatenate(
        [np.arange(s0, min(s0 + 64, s1)) for s0, s1 in bounds] + [np.arange(s1 - 64, s1) for s0, s1 in bounds]))
    O_full, L_full = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e_full, rows=rows,
                                     gemm_dtype=np.float32 if big else np.float64)
    for r, (s0, s1) in enumerate(bounds):
        out = cp.compact_and_attend(ps[r], s0, allc[:r] if r else None, Q[:, :, s0:s1].contiguous(),
                                    K[:, :, s0:s1].contiguous(), V[:, :, s0:s1].contiguous(),
                                    delta[:, :, s0:s1].contiguous())
        torch.cuda.synchronize()
        assert int(out["status_word"].view(torch.int32).item()) == 0
        Kc, Vc, dc, P, pc = oracle.cp_compact([c[1] for c in cands[:r]], s0, d32[:, :, s0:s1], I.K[:, :, s0:s1],
                                              I.V[:, :, s0:s1], w_heads, wl.w)
        assert out["prefix_rows"] == P
        np.testing.assert_array_equal(out["pos_c"].cpu().numpy(), pc)
        np.testing.assert_array_equal(out["delta_c"].cpu().numpy(), dc)
        np.testing.assert_array_equal(to_np(out["Kc"]), Kc)
        np.testing.assert_array_equal(to_np(out["Vc"]), Vc)
        ec = oracle.topw_eviction_heads(dc, np.full(wl.H, wl.w) if w_heads is None else w_heads, wl.w)
        np.testing.assert_array_equal(out["evict"].cpu().numpy(), ec)
        own = (rows >= s0) & (rows < s1)
        assert_close(to_np(out["LSE"])[:, :, rows[own] - s0], L_full[:, :, rows[own]], f"LSE shard {r}")
        assert_close(to_np(out["O"])[:, :, rows[own] - s0], O_full[:, :, rows[own]], f"O shard {r}")


def _bits_rows(I, name, ref, wl):
    """bf16 bits of the candidate rows the oracle picked (zero past a row's count)."""
    G = wl.H // wl.Hkv
    bits = I.bits[name]
    out = np.zeros((wl.B, wl.H, wl.w, wl.d), dtype=np.uint16)
    for b in range(wl.B):
        for h in range(wl.H):
            pos = ref["pos"][b, h]
            k = int((pos >= 0).sum())
            out[b, h, :k] = bits[b, h // G, pos[:k]]
    return out
