"""Pins of the oracle's context-parallel prefill (each rank holds one contiguous
shard of the sequence and receives, in one exchange, the best keys of every
earlier shard; "Future Directions" of the page "Trainable Dynamic Mask Sparse
Attention" names long-context scaling, the exchange follows from the m_t
equation: the best keys of a union are among the best keys of its parts).

Pinned against the whole-sequence definition, not against itself: for every
shard, the selection of its queries computed on the compacted sequence, mapped
back to original positions, equals the whole-sequence selection bit for bit,
and the attention of its queries equals the whole-sequence attention rows."""
import math

import numpy as np
import pytest

import oracle
from workloads import get, make_delta, make_inputs


def _whole(I, d32, w_heads, w):
    e = oracle.topw_eviction_heads(d32, np.full(d32.shape[1], w) if w_heads is None else w_heads, w)
    O, L = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e)
    return e, O, L


def _run_rank(I, d32, bounds, r, w_heads, w):
    """Rank r of the sharded computation, from the candidates of the shards before it."""
    cands = []
    for q in range(r):
        s0, s1 = bounds[q]
        cands.append(oracle.cp_candidates(d32[:, :, s0:s1], I.K[:, :, s0:s1], I.V[:, :, s0:s1], w_heads, w, s0))
    s0, s1 = bounds[r]
    Kc, Vc, dc, P, pc = oracle.cp_compact(cands, s0, d32[:, :, s0:s1], I.K[:, :, s0:s1], I.V[:, :, s0:s1],
                                          w_heads, w)
    H = d32.shape[1]
    ec = oracle.topw_eviction_heads(dc, np.full(H, w) if w_heads is None else w_heads, w)
    O, L = oracle.attn_fwd(I.Q[:, :, s0:s1], Kc, Vc, dc.astype(np.float64), ec, q_pos0=P)
    return Kc, Vc, dc, P, pc, ec, O, L


@pytest.mark.parametrize("R", [2, 3, 4])
@pytest.mark.parametrize("w,w_heads", [(37, None), (300, None), (1000, None), (120, [120, 5, 64, 1])])
def test_sharded_equals_whole_sequence(R, w, w_heads):
    wl = get("tiny").with_(B=2, H=4, Hkv=2, N=600, d=16, w=w, dtype="f32", seed=R * 100 + w)
    I = make_inputs(wl)
    _, d = oracle.gate(I.V, I.Delta, I.A)
    d32 = d.astype(np.float32)
    e_full, O_full, L_full = _whole(I, d32, w_heads, w)
    bounds = oracle.cp_shard_bounds(wl.N, R)
    G = wl.G
    for r in range(R):
        s0, s1 = bounds[r]
        Kc, Vc, dc, P, pc, ec, O, L = _run_rank(I, d32, bounds, r, w_heads, w)
        assert P == min(G * w, s0)
        # selection of every own query, mapped back to original positions
        for b in range(wl.B):
            for h in range(wl.H):
                g = h // G
                Mc = oracle.mask_from_eviction(ec[b, h], np.arange(P, P + s1 - s0))   # [own queries, P + len]
                Mf = oracle.mask_from_eviction(e_full[b, h], np.arange(s0, s1))      # [own queries, N]
                for i in range(s1 - s0):
                    got = np.sort(pc[b, g, np.nonzero(Mc[i])[0]])
                    assert (got >= 0).all()
                    np.testing.assert_array_equal(got, np.nonzero(Mf[i])[0])
        np.testing.assert_allclose(O, O_full[:, :, s0:s1], rtol=0, atol=1e-12)
        np.testing.assert_allclose(L, L_full[:, :, s0:s1], rtol=0, atol=1e-12)


def test_candidates_are_the_best_keys_of_the_shard():
    rng = np.random.default_rng(7)
    B, H, Hkv, L, d, w = 1, 2, 1, 50, 4, 9
    delta = np.round(rng.random((B, H, L)).astype(np.float32) * 5) / 5   # ties
    K = rng.standard_normal((B, Hkv, L, d)).astype(np.float32)
    V = rng.standard_normal((B, Hkv, L, d)).astype(np.float32)
    c = oracle.cp_candidates(delta, K, V, [9, 3], w, 1000)
    for h, wh in enumerate([9, 3]):
        order = sorted(range(L), key=lambda j: (-float(delta[0, h, j]), j))[:wh]
        np.testing.assert_array_equal(c["pos"][0, h, :wh], 1000 + np.sort(order))
        assert (c["pos"][0, h, wh:] == -1).all() and np.isneginf(c["delta"][0, h, wh:]).all()
        np.testing.assert_array_equal(c["K"][0, h, :wh], K[0, 0, np.sort(order)])


def test_short_prefix_is_kept_whole():
    """A prefix shorter than the window: every prefix key is a candidate of every head, so the
    compacted sequence is the original one (no padding, true delta for every head)."""
    wl = get("tiny").with_(B=1, H=2, Hkv=1, N=90, d=8, w=64, dtype="f32", seed=3)
    I = make_inputs(wl)
    _, d = oracle.gate(I.V, I.Delta, I.A)
    d32 = d.astype(np.float32)
    bounds = oracle.cp_shard_bounds(90, 2)
    Kc, Vc, dc, P, pc, ec, O, L = _run_rank(I, d32, bounds, 1, None, 64)
    assert P == 45
    np.testing.assert_array_equal(pc[0, 0], np.arange(90))
    np.testing.assert_array_equal(dc, d32)
    np.testing.assert_array_equal(Kc, I.K)
