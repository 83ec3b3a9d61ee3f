"""Pins of the oracle's masked attention (forward, backward) and decode.

Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Efficient
Sparse Attention Computation" (equation for o_t) and "Theoretical Guarantees
for Safe Computation Skipping" (masked pairs: zero weight, zero gradient).
Reading of the garbled operator: the mask is added to q k^T / sqrt(d) --
selected keys get +delta_j, others -inf.

Pins: w >= N reduces to dense causal attention with an additive float bias,
checked against torch's scaled_dot_product_attention (and its autograd) in
float64; strictly increasing delta reduces to sliding-window attention; a
zero query gives closed-form outputs; central finite differences pin the
analytic backward; invariants (masked keys have no influence, sum of
ddelta is zero per row set).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import get, make_delta, make_inputs


def _rand(seed, B=2, H=4, Hkv=2, N=24, d=8):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, H, N, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    return Q, K, V


def _evict(delta, w):
    B, H, N = delta.shape
    return np.stack([np.stack([oracle.topw_eviction(delta[b, h].astype(np.float32), w)
                               for h in range(H)]) for b in range(B)])


def _sdpa(Q, K, V, bias_mask, scale):
    """torch SDPA, float64, K/V repeated over the query heads of each group."""
    G = Q.shape[1] // K.shape[1]
    q = torch.from_numpy(Q)
    k = torch.from_numpy(K).repeat_interleave(G, dim=1)
    v = torch.from_numpy(V).repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=torch.from_numpy(bias_mask), scale=scale)


def test_full_window_is_dense_causal_attention_with_bias():
    Q, K, V = _rand(0)
    B, H, N, d = Q.shape
    delta = make_delta((B, H, N), seed=1).astype(np.float64)
    e = _evict(delta, N)          # w = N: all causal keys
    scale = 1.0 / math.sqrt(d)
    O, LSE = oracle.attn_fwd(Q, K, V, delta, e)
    causal = np.tril(np.ones((N, N), dtype=bool))
    bias = np.where(causal[None, None], delta[:, :, None, :], -np.inf)
    ref = _sdpa(Q, K, V, bias, scale).numpy()
    np.testing.assert_allclose(O, ref, rtol=1e-12, atol=1e-12)


def test_increasing_delta_is_sliding_window_attention():
    Q, K, V = _rand(1, N=40)
    B, H, N, d = Q.shape
    w = 7
    delta = make_delta((B, H, N), seed=0, kind="increasing").astype(np.float64)
    e = _evict(delta, w)
    O, _ = oracle.attn_fwd(Q, K, V, delta, e)
    t = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    window = (j <= t) & (j > t - w)
    bias = np.where(window[None, None], delta[:, :, None, :], -np.inf)
    ref = _sdpa(Q, K, V, bias, 1.0 / math.sqrt(d)).numpy()
    np.testing.assert_allclose(O, ref, rtol=1e-12, atol=1e-12)


def test_zero_query_constant_delta_closed_form():
    """q = 0 and delta = c: every selected key has weight 1/|S_t| with
    |S_t| = min(t+1, w) and S_t = {0..min(t, w-1)} (all ties -> lowest
    indices), so O_t is the mean of those v_j and LSE_t = c + ln |S_t|."""
    B, H, Hkv, N, d, w = 1, 2, 1, 30, 4, 9
    rng = np.random.default_rng(3)
    Q = np.zeros((B, H, N, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    c = 0.375
    delta = np.full((B, H, N), c)
    e = _evict(delta, w)
    O, LSE = oracle.attn_fwd(Q, K, V, delta, e)
    for t in range(N):
        n = min(t + 1, w)
        np.testing.assert_allclose(O[0, :, t], np.broadcast_to(V[0, 0, :n].mean(axis=0), (H, d)), rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(LSE[0, :, t], c + math.log(n), rtol=1e-14)


def test_masked_keys_have_no_influence():
    """Changing K and V rows of keys a query does not select leaves its output
    bit-for-bit unchanged (exact zero weight)."""
    Q, K, V = _rand(4, B=1, H=2, Hkv=1, N=32)
    delta = make_delta((1, 2, 32), seed=4).astype(np.float64)
    w = 6
    e = _evict(delta, w)
    O, LSE = oracle.attn_fwd(Q, K, V, delta, e)
    t = 31
    sel = (np.arange(32) <= t) & (t < e[0, 0])
    K2, V2 = K.copy(), V.copy()
    K2[0, 0, ~sel] += 100.0
    V2[0, 0, ~sel] -= 100.0
    O2, LSE2 = oracle.attn_fwd(Q, K2, V2, delta, e)
    assert np.array_equal(O[0, 0, t], O2[0, 0, t]) and LSE[0, 0, t] == LSE2[0, 0, t]


def test_rows_subset_matches_full():
    Q, K, V = _rand(5, N=50)
    delta = make_delta(Q.shape[:3], seed=5).astype(np.float64)
    e = _evict(delta, 11)
    O, LSE = oracle.attn_fwd(Q, K, V, delta, e)
    rows = np.array([0, 7, 13, 49])
    O2, LSE2 = oracle.attn_fwd(Q, K, V, delta, e, rows=rows)
    np.testing.assert_array_equal(O2[:, :, rows], O[:, :, rows])
    np.testing.assert_array_equal(LSE2[:, :, rows], LSE[:, :, rows])


def _loss(Q, K, V, delta, e, dO):
    O, _ = oracle.attn_fwd(Q, K, V, delta, e)
    return float((O * dO).sum())


@pytest.mark.parametrize("w", [3, 16])
def test_backward_matches_central_differences(w):
    Q, K, V = _rand(6, B=1, H=2, Hkv=1, N=12, d=4)
    rng = np.random.default_rng(9)
    dO = rng.standard_normal(Q.shape)
    delta = rng.uniform(0.2, 1.0, size=Q.shape[:3])
    e = _evict(delta, w)   # selection held constant under the perturbation
    dQ, dK, dV, dd = oracle.attn_bwd(Q, K, V, delta, e, dO)
    eps = 1e-6
    for name, X, G in (("Q", Q, dQ), ("K", K, dK), ("V", V, dV), ("delta", delta, dd)):
        num = np.zeros_like(X)
        it = np.nditer(X, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            Xp = X.copy(); Xp[i] += eps
            Xm = X.copy(); Xm[i] -= eps
            args = {"Q": Q, "K": K, "V": V, "delta": delta}
            args[name] = Xp
            fp = _loss(args["Q"], args["K"], args["V"], args["delta"], e, dO)
            args[name] = Xm
            fm = _loss(args["Q"], args["K"], args["V"], args["delta"], e, dO)
            num[i] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(G, num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_backward_full_window_matches_torch_autograd():
    Q, K, V = _rand(7, N=20)
    B, H, N, d = Q.shape
    rng = np.random.default_rng(8)
    dO = rng.standard_normal(Q.shape)
    delta = rng.uniform(0.1, 1.0, size=(B, H, N))
    e = _evict(delta, N)
    dQ, dK, dV, dd = oracle.attn_bwd(Q, K, V, delta, e, dO)
    G = H // K.shape[1]
    q = torch.from_numpy(Q).requires_grad_()
    k = torch.from_numpy(K).requires_grad_()
    v = torch.from_numpy(V).requires_grad_()
    dl = torch.from_numpy(delta).requires_grad_()
    causal = torch.tril(torch.ones(N, N, dtype=torch.bool))
    bias = torch.where(causal, dl[:, :, None, :], torch.tensor(-math.inf, dtype=torch.float64))
    out = torch.nn.functional.scaled_dot_product_attention(
        q, k.repeat_interleave(G, 1), v.repeat_interleave(G, 1), attn_mask=bias, scale=1 / math.sqrt(d))
    out.backward(torch.from_numpy(dO))
    np.testing.assert_allclose(dQ, q.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK, k.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dV, v.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dd, dl.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_invariants():
    Q, K, V = _rand(10, B=1, H=2, Hkv=1, N=40)
    rng = np.random.default_rng(10)
    dO = rng.standard_normal(Q.shape)
    delta = make_delta((1, 2, 40), seed=10, kind="levels", levels=6).astype(np.float64)
    e = _evict(delta, 5)
    dQ, dK, dV, dd = oracle.attn_bwd(Q, K, V, delta, e, dO)
    # softmax shift invariance: each row of dS sums to zero, hence so does ddelta
    np.testing.assert_allclose(dd.sum(axis=-1), 0.0, atol=1e-12)
    # keys selected by no query (of any head in the group) get exactly zero dK, dV
    never = np.ones(40, dtype=bool)
    for h in range(2):
        never &= e[0, h] == np.arange(40)
    assert never.any()
    assert np.all(dK[0, 0, never] == 0) and np.all(dV[0, 0, never] == 0)
    for h in range(2):
        nh = e[0, h] == np.arange(40)
        assert np.all(dd[0, h, nh] == 0)


# ---------------------------------------------------------------- gate backward

def test_gate_backward_matches_central_differences():
    rng = np.random.default_rng(12)
    B, Hkv, N, d, H = 2, 2, 5, 3, 4
    V = rng.standard_normal((B, Hkv, N, d))
    Delta = rng.standard_normal((Hkv * d, H)) * 0.3
    A = rng.uniform(-1, 0, size=H)
    dd = rng.standard_normal((B, H, N))
    dDelta, dA, dVg = oracle.gate_bwd(V, Delta, A, dd)

    def L(V_, D_, A_):
        return float((oracle.gate(V_, D_, A_)[1] * dd).sum())

    eps = 1e-6
    for name, X, G in (("V", V, dVg), ("Delta", Delta, dDelta), ("A", A, dA)):
        num = np.zeros_like(X)
        it = np.nditer(X, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            args = {"V": V, "Delta": Delta, "A": A}
            Xp = X.copy(); Xp[i] += eps
            Xm = X.copy(); Xm[i] -= eps
            args[name] = Xp
            fp = L(args["V"], args["Delta"], args["A"])
            args[name] = Xm
            fm = L(args["V"], args["Delta"], args["A"])
            num[i] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(G, num, rtol=1e-6, atol=1e-9, err_msg=name)


# ---------------------------------------------------------------- decode

def test_decode_select_is_last_row_of_the_selection():
    B, H, L, w = 2, 3, 120, 17
    for kind in ("uniform", "levels", "constant"):
        delta = make_delta((B, H, L), seed=21, kind=kind, levels=5)
        sel = oracle.decode_select(delta, w)
        for b in range(B):
            for h in range(H):
                e = oracle.topw_eviction(delta[b, h], w)
                np.testing.assert_array_equal(sel[b, h], np.nonzero(e > L - 1)[0])
                M = oracle.topw_sets_bruteforce(delta[b, h], w)
                np.testing.assert_array_equal(sel[b, h], np.nonzero(M[L - 1])[0])


def test_decode_select_append_equals_the_full_selection_at_every_length():
    # growing the cache key by key from one key, across the point where min(L, w) stops growing,
    # on uniform, heavily tied and constant gate values (ties test the lower-index-first rule)
    B, H, L, w = 2, 3, 90, 16
    for kind in ("uniform", "levels", "constant"):
        delta = make_delta((B, H, L), seed=33, kind=kind, levels=4)
        sel = oracle.decode_select(delta[:, :, :1], w)
        for n in range(2, L + 1):
            sel = oracle.decode_select_append(sel, delta[:, :, :n], w)
            np.testing.assert_array_equal(sel, oracle.decode_select(delta[:, :, :n], w), err_msg=f"{kind} L={n}")


def test_decode_select_append_cases():
    # hand-checked: w = 3, delta of keys 0..3 = [0.5, 0.2, 0.9, x]
    d = np.array([[[0.5, 0.2, 0.9, 0.0]]], dtype=np.float32)
    prev = np.array([[[0, 1, 2]]])
    for x, want in ((0.1, [0, 1, 2]), (0.2, [0, 1, 2]), (0.3, [0, 2, 3]), (1.0, [0, 2, 3])):
        d[0, 0, 3] = x
        np.testing.assert_array_equal(oracle.decode_select_append(prev, d, 3)[0, 0], want, err_msg=str(x))
    # equal worst values: the larger index is the worst (key 2 goes, not key 1)
    d = np.array([[[0.9, 0.2, 0.2, 0.5]]], dtype=np.float32)
    np.testing.assert_array_equal(oracle.decode_select_append(np.array([[[0, 1, 2]]]), d, 3)[0, 0], [0, 1, 3])


def test_chunked_queries_are_rows_of_the_full_sequence():
    # a chunk of queries at an offset sees the same keys and selection as those rows of the whole
    # sequence; the last row also equals decode
    Q, K, V = _rand(17, B=1, H=4, Hkv=2, N=90, d=8)
    delta = make_delta(Q.shape[:3], seed=17).astype(np.float64)
    w = 12
    e = _evict(delta, w)
    O, LSE = oracle.attn_fwd(Q, K, V, delta, e)
    for q0 in (1, 37, 89):
        Oc, Lc = oracle.attn_fwd(Q[:, :, q0:], K, V, delta, e, q_pos0=q0)
        np.testing.assert_allclose(Oc, O[:, :, q0:], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(Lc, LSE[:, :, q0:], rtol=1e-14)


def test_decode_attn_is_last_row_of_prefill():
    Q, K, V = _rand(13, B=2, H=4, Hkv=2, N=64, d=8)
    delta = make_delta(Q.shape[:3], seed=13).astype(np.float64)
    w = 10
    e = _evict(delta, w)
    O, LSE = oracle.attn_fwd(Q, K, V, delta, e)
    sel = oracle.decode_select(delta.astype(np.float32), w)
    o, lse = oracle.decode_attn(Q[:, :, -1:, :], K, V, delta, sel)
    np.testing.assert_allclose(o, O[:, :, -1], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, LSE[:, :, -1], rtol=1e-14)


# ---------------------------------------------------------------- end to end on tiny

def test_tiny_workload_chain_runs_and_rows_sum_to_one():
    wl = get("tiny")
    I = make_inputs(wl)
    _, delta = oracle.gate(I.V, I.Delta, I.A)
    d32 = delta.astype(np.float32)
    e = _evict(d32, wl.w)
    # the mask keeps exactly min(t+1, w) keys per row
    for h in range(wl.H):
        M = oracle.mask_from_eviction(e[0, h])
        np.testing.assert_array_equal(M.sum(axis=1), np.minimum(np.arange(wl.N) + 1, wl.w))
    assert sum(int(oracle.mask_from_eviction(e[0, h]).sum()) for h in range(wl.H)) == wl.kept_pairs()
    # all-ones V: every output entry is exactly a convex combination of ones
    O, _ = oracle.attn_fwd(I.Q, I.K, np.ones_like(I.V), d32.astype(np.float64), e)
    np.testing.assert_allclose(O, 1.0, rtol=1e-13)
