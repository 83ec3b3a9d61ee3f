"""Pins of the oracle's causal top-w selection m_t = f(top_w(delta + m_c^t)).

Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Dynamic
Sparse Mask Generation", equation for m_t.  Readings: ties go to the lower key
index; a row with fewer than w causal keys keeps all of them; the query's own
key competes like any other.

The sequential eviction pass is pinned against the per-query brute force, a
worked example derived by hand, closed forms of special inputs, and the
structural invariants (|S_t| = min(t+1, w), S_{t+1} within S_t + {t+1}, each
key selected on an interval of queries starting at the key).
"""
import numpy as np
import pytest

import oracle
from workloads import make_delta


def test_worked_example_by_hand():
    # delta = [0.5, 0.9, 0.5, 0.7, 0.9, 0.1], w = 2, order (delta desc, index asc):
    #  t=0: {0}           t=1: {0,1}
    #  t=2: best of {0:.5, 1:.9, 2:.5} -> 1, then the 0.5 tie goes to key 0 -> {0,1};
    #       key 2 is never selected: e_2 = 2
    #  t=3: {1:.9, 3:.7} -> key 0 leaves: e_0 = 3
    #  t=4: {1:.9, 4:.9} -> key 3 leaves: e_3 = 4
    #  t=5: 0.1 never enters: e_5 = 5;  keys 1 and 4 stay to the end: e = N = 6
    delta = np.array([0.5, 0.9, 0.5, 0.7, 0.9, 0.1], dtype=np.float32)
    e = oracle.topw_eviction(delta, 2)
    np.testing.assert_array_equal(e, [3, 6, 2, 4, 6, 5])
    M = oracle.topw_sets_bruteforce(delta, 2)
    expect_sets = [{0}, {0, 1}, {0, 1}, {1, 3}, {1, 4}, {1, 4}]
    for t in range(6):
        assert set(np.nonzero(M[t])[0]) == expect_sets[t]


@pytest.mark.parametrize("kind,levels", [("uniform", 0), ("levels", 3), ("levels", 7), ("constant", 0)])
@pytest.mark.parametrize("N,w", [(1, 1), (7, 1), (17, 4), (40, 9), (64, 63), (64, 64), (50, 80)])
def test_eviction_pass_equals_brute_force(kind, levels, N, w):
    for seed in range(3):
        delta = make_delta((N,), seed=seed * 31 + N, kind=kind, levels=levels)
        M = oracle.topw_sets_bruteforce(delta, w)
        e = oracle.topw_eviction(delta, w)
        np.testing.assert_array_equal(oracle.mask_from_eviction(e), M)
        # the brute-force mask has the interval form and encodes the same e
        np.testing.assert_array_equal(oracle.eviction_from_mask(M), e)


@pytest.mark.parametrize("N,w", [(33, 5), (64, 16), (100, 100)])
def test_invariants(N, w):
    delta = make_delta((N,), seed=11, kind="levels", levels=5)
    M = oracle.topw_sets_bruteforce(delta, w)
    for t in range(N):
        assert M[t].sum() == min(t + 1, w)
        assert not M[t, t + 1:].any()             # causal
        if t + 1 < N:
            new = M[t + 1] & ~M[t]
            assert (np.nonzero(new)[0] <= t + 1).all() and new.sum() <= 1
            assert not new[: t + 1].any()          # only key t+1 can join


def test_strictly_increasing_delta_is_sliding_window():
    N, w = 300, 37
    delta = make_delta((N,), seed=0, kind="increasing")
    e = oracle.topw_eviction(delta, w)
    np.testing.assert_array_equal(e, np.minimum(np.arange(N) + w, N))


@pytest.mark.parametrize("kind", ["decreasing", "constant"])
def test_decreasing_or_constant_delta_keeps_the_prefix(kind):
    """Decreasing delta, or all ties broken toward the lower index: the
    selection is {0 .. min(t, w-1)} -- keys below w are never evicted, later
    keys never enter."""
    N, w = 200, 23
    delta = make_delta((N,), seed=0, kind=kind)
    e = oracle.topw_eviction(delta, w)
    j = np.arange(N)
    np.testing.assert_array_equal(e, np.where(j < w, N, j))


def test_window_at_least_N_keeps_all_causal_keys():
    N = 90
    delta = make_delta((N,), seed=5, kind="uniform")
    for w in (N, N + 1, 10 * N):
        np.testing.assert_array_equal(oracle.topw_eviction(delta, w), np.full(N, N))


@pytest.mark.parametrize("N,w", [(203, 31), (203, 500), (100, 16), (64, 64)])
def test_live_keys_per_block_against_mask(N, w):
    Bq = 16
    for kind in ("uniform", "levels", "increasing", "constant"):
        delta = make_delta((N,), seed=2, kind=kind, levels=4)
        M = oracle.topw_sets_bruteforce(delta, w)
        e = oracle.topw_eviction(delta, w)
        blocks = oracle.live_keys_per_block(e, Bq)
        assert len(blocks) == (N + Bq - 1) // Bq
        for bi, (full, partial) in enumerate(blocks):
            t0, t1 = bi * Bq, min(bi * Bq + Bq, N)
            union = M[t0:t1].any(axis=0)
            inter = M[t0:t1].all(axis=0)
            np.testing.assert_array_equal(np.sort(np.concatenate([full, partial])), np.nonzero(union)[0])
            np.testing.assert_array_equal(full, np.nonzero(inter)[0])
            assert set(full).isdisjoint(partial)
            # the live set never exceeds w + Bq keys, the partial keys never 2 Bq
            assert full.size + partial.size <= w + Bq
            assert partial.size <= 2 * Bq


# ---------------------------------------------------------------- per-head windows

def test_head_windows_clamp():
    np.testing.assert_array_equal(oracle.head_windows([0, 1, 5, 9, 100], 9), [1, 1, 5, 9, 9])


@pytest.mark.parametrize("kind,levels", [("uniform", 0), ("levels", 4), ("constant", 0)])
def test_eviction_heads_equals_brute_force_per_head(kind, levels):
    """Each head's mask is the brute-force selection with that head's own window
    (windows below, at and above the row length; one above the largest window is
    clamped to it)."""
    N, w = 37, 30
    w_heads = [1, 4, 13, 30, 45]
    d = make_delta((2, len(w_heads), N), seed=91, kind=kind, levels=levels)
    e = oracle.topw_eviction_heads(d, w_heads, w)
    eff = [1, 4, 13, 30, 30]
    for b in range(2):
        for h, wh in enumerate(eff):
            M = oracle.topw_sets_bruteforce(d[b, h], wh)
            np.testing.assert_array_equal(oracle.mask_from_eviction(e[b, h]), M)
            assert (M.sum(axis=1) == np.minimum(np.arange(N) + 1, wh)).all()


def test_eviction_heads_increasing_is_a_window_per_head():
    """Strictly increasing delta: head h attends to the sliding window of its
    own width W_h, [t - W_h + 1, t]."""
    N = 50
    w_heads = [3, 11, 50]
    d = make_delta((1, 3, N), seed=0, kind="increasing")
    e = oracle.topw_eviction_heads(d, w_heads, 50)
    for h, wh in enumerate(w_heads):
        expect = np.minimum(np.arange(N) + wh, N)
        np.testing.assert_array_equal(e[0, h], expect)


def test_decode_select_heads_by_sorting():
    """Row (b, h) holds the min(L, W_h) best keys by (delta desc, index asc), ascending."""
    rng = np.random.default_rng(5)
    B, H, L, w = 2, 3, 40, 25
    d = np.round(rng.random((B, H, L)).astype(np.float32) * 8) / 8   # many ties
    w_heads = [25, 2, 60]
    rows = oracle.decode_select_heads(d, w_heads, w)
    eff = [25, 2, 25]
    for b in range(B):
        for h in range(H):
            order = sorted(range(L), key=lambda j: (-float(d[b, h, j]), j))
            np.testing.assert_array_equal(rows[b * H + h], sorted(order[:min(L, eff[h])]))
