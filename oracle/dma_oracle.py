"""Plain CPU oracle for the Dynamic Mask Attention (DMA) hot path.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA library and never calls it; it is deliberately slow and written to be
checked by eye against the method's definition on the page "Trainable Dynamic
Mask Sparse Attention: Bridging Efficiency and Effectiveness in Long-Context
Language Models" (Hugging Face blog "dmattn"):

  * gate      -- section "Dynamic Sparse Mask Generation", equation for delta
                 ("Dynamic Weight Computation"): delta = exp(tau(v Delta) x A);
  * selection -- same section, equation for m_t ("Mask Combination with Causal
                 Constraints"): m_t = f(top_w(delta + m_c^t));
  * attention -- section "Efficient Sparse Attention Computation", equation for
                 o_t: o_t = softmax(q_t k^T / sqrt(d_h) (+) m_t) v;
  * backward  -- "Theoretical Guarantees for Safe Computation Skipping" (masked
                 pairs give exactly zero weight and zero gradient) and
                 "Gradient Flow Integrity" (end-to-end trainable).

Readings where the page is silent or garbled (each repeated where it is used):
  tau = softplus; v at key position j is the concatenation of the Hkv key/value
  heads (length Hkv*d), Delta is [Hkv*d, H], and delta is per query head;
  the mask is ADDED to the scaled scores (selected key j contributes
  +delta_j, others -inf); top-w orders keys by delta descending and breaks ties
  toward the lower key index; a row with fewer than w causal keys keeps all of
  them; the selection is a constant in the backward pass; LSE is the natural
  log of the softmax denominator.

Precision: float64 throughout unless a caller asks for float32 GEMMs on large
inputs (reductions stay in float64).

Parity pins: see tests/test_oracle_*.py.  Every function below is pinned by a
test that does not re-type its formula (brute force, closed forms, library
routines on special cases, finite differences, invariants).
"""
from __future__ import annotations

import heapq
import math

import numpy as np

__all__ = [
    "softplus",
    "sigmoid",
    "gate",
    "topw_sets_bruteforce",
    "topw_eviction",
    "mask_from_eviction",
    "eviction_from_mask",
    "live_keys_per_block",
    "attn_fwd",
    "attn_bwd",
    "gate_bwd",
    "decode_select",
    "decode_select_append",
    "decode_attn",
    "head_windows",
    "topw_eviction_heads",
    "decode_select_heads",
    "cp_candidates",
    "cp_prefix_len",
    "cp_compact",
    "cp_shard_bounds",
]


# ----------------------------------------------------------------------------
# Gate: delta = exp(tau(v Delta) * A), tau = softplus
# ----------------------------------------------------------------------------

def softplus(x: np.ndarray) -> np.ndarray:
    """tau(x) = ln(1 + e^x), the non-negative function of the delta equation
    (reading: softplus).  Written in the overflow-free form
    max(x, 0) + ln(1 + e^{-|x|})."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def sigmoid(x: np.ndarray) -> np.ndarray:
    """Derivative of softplus, 1 / (1 + e^{-x}), evaluated without overflow."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def gate(V: np.ndarray, Delta: np.ndarray, A: np.ndarray, gemm_dtype=np.float64):
    """Content-aware gate ("Dynamic Weight Computation" equation).

    V      [B, Hkv, N, d]  value vectors.
    Delta  [Hkv*d, H]      learnable sampling weights.
    A      [H]             per-head selective control.

    Reading: the value vector of key position j is the concatenation over the
    Hkv heads, v_j[g*d + c] = V[b, g, j, c]; x = v Delta is [B, N, H];
    delta = exp(A_h * softplus(x)) is one value per (batch, query head, key).

    Returns (x, delta), both [B, H, N] float64.
    """
    B, Hkv, N, d = V.shape
    H = Delta.shape[1]
    assert Delta.shape == (Hkv * d, H)
    v = np.asarray(V, dtype=gemm_dtype).transpose(0, 2, 1, 3).reshape(B, N, Hkv * d)
    x = np.matmul(v, np.asarray(Delta, dtype=gemm_dtype)).astype(np.float64)  # [B, N, H]
    x = x.transpose(0, 2, 1).copy()  # [B, H, N]
    delta = np.exp(np.asarray(A, dtype=np.float64)[None, :, None] * softplus(x))
    return x, delta


# ----------------------------------------------------------------------------
# Causal top-w selection: m_t = f(top_w(delta + m_c^t))
# ----------------------------------------------------------------------------

def _better(di: float, i: int, dj: float, j: int) -> bool:
    """Total order of the top-w selection: larger delta first; equal delta ->
    lower key index first (tie reading)."""
    return di > dj or (di == dj and i < j)


def topw_sets_bruteforce(delta_row: np.ndarray, w: int) -> np.ndarray:
    """Selection by the definition, one query at a time.

    For query t the causal constraint m_c^t removes keys j > t; top_w keeps
    the min(t+1, w) best of the remaining keys; f sends every other key to
    -inf.  Returns the boolean mask M[t, j] (True = selected).  O(N^2 log N):
    for tiny inputs only.
    """
    d = [float(v) for v in np.asarray(delta_row, dtype=np.float32)]
    N = len(d)
    M = np.zeros((N, N), dtype=bool)
    for t in range(N):
        order = sorted(range(t + 1), key=lambda j: (-d[j], j))
        for j in order[: min(t + 1, w)]:
            M[t, j] = True
    return M


def topw_eviction(delta_row: np.ndarray, w: int) -> np.ndarray:
    """Eviction index of every key, from one sequential pass.

    Because delta depends on the key but not on the query, the rank of key j
    among keys 0..t can only grow with t, so key j is selected exactly for the
    queries t in [j, e_j).  The pass keeps the current selection in a min-heap
    ordered by the selection order; after key t is pushed the worst member is
    popped whenever the heap holds more than w keys, and that key's e is t.
    Keys never popped get e = N.  e_j == j means key j is never selected.
    """
    d = np.asarray(delta_row, dtype=np.float32)
    N = d.shape[0]
    e = np.full(N, N, dtype=np.int64)
    heap: list[tuple[float, int]] = []   # (delta, -j): smallest = worst
    for t in range(N):
        heapq.heappush(heap, (float(d[t]), -t))
        if len(heap) > w:
            _, negj = heapq.heappop(heap)
            e[-negj] = t
    return e


def mask_from_eviction(e: np.ndarray, q_rows: np.ndarray | None = None) -> np.ndarray:
    """M[t, j] = (j <= t < e_j) for the query rows q_rows (default 0..N-1)."""
    N = e.shape[-1]
    t = np.arange(N) if q_rows is None else np.asarray(q_rows)
    j = np.arange(N)
    return (j[None, :] <= t[:, None]) & (t[:, None] < e[None, :])


def eviction_from_mask(M: np.ndarray) -> np.ndarray:
    """Inverse of mask_from_eviction for a full [N, N] mask that has the
    interval form; raises if some key's selected queries are not an interval
    starting at the key itself."""
    N = M.shape[0]
    e = np.empty(N, dtype=np.int64)
    for j in range(N):
        col = M[:, j]
        ts = np.nonzero(col)[0]
        if ts.size == 0:
            e[j] = j
            continue
        if ts[0] != j or ts[-1] - ts[0] + 1 != ts.size:
            raise ValueError(f"key {j}: selected queries are not an interval from j")
        e[j] = ts[-1] + 1
    return e


def live_keys_per_block(e: np.ndarray, Bq: int):
    """Keys a query block [t0, t0+Bq) attends to, split into 'full' keys
    (selected by every query row of the block) and 'partial' keys.

    Returns a list over blocks of (full: sorted int array, partial: sorted int
    array).  A key is full when every existing row of the block selects it:
    j <= t0 and e_j >= t1 with t1 = min(t0 + Bq, N) (rows past N do not exist).
    """
    N = e.shape[0]
    j = np.arange(N)
    out = []
    for t0 in range(0, N, Bq):
        t1 = min(t0 + Bq, N)
        live = (j < t1) & (e > np.maximum(j, t0))
        full = live & (j <= t0) & (e >= t1)
        out.append((np.nonzero(full)[0], np.nonzero(live & ~full)[0]))
    return out


# ----------------------------------------------------------------------------
# Masked attention forward / backward
# ----------------------------------------------------------------------------

def _scores(Qh, Kg, delta_h, e_h, rows, scale, gemm_dtype, q_pos0=0):
    """Scaled scores plus the additive mask of rows `rows` (query row i sits
    at position q_pos0 + i).

    Reading of the garbled operator in the o_t equation: the mask m_t is added
    to q_t k^T / sqrt(d): selected key j contributes +delta_j, non-selected
    keys -inf (f of the m_t equation)."""
    N = Kg.shape[0]
    s = np.matmul(np.asarray(Qh[rows], dtype=gemm_dtype),
                  np.asarray(Kg, dtype=gemm_dtype).T).astype(np.float64) * scale
    s = s + np.asarray(delta_h, dtype=np.float64)[None, :]
    t = q_pos0 + (np.asarray(rows)[:, None] if rows is not None else np.arange(Qh.shape[0])[:, None])
    j = np.arange(N)[None, :]
    sel = (j <= t) & (t < np.asarray(e_h)[None, :])
    return np.where(sel, s, -np.inf), sel


def attn_fwd(Q, K, V, delta, evict, scale=None, q_pos0: int = 0, rows=None,
             gemm_dtype=np.float64, chunk: int = 1024):
    """Masked attention forward ("Efficient Sparse Attention Computation").

    Q [B, H, Nq, d] (query row i sits at position q_pos0 + i), K, V
    [B, Hkv, N, d], delta [B, H, N], evict [B, H, N] (the selection as
    eviction indices).  Returns O [B, H, Nq, d] and LSE [B, H, Nq] (natural log
    of the softmax denominator), float64.  `rows` restricts the computation to
    a subset of query rows (other rows are NaN).

    Dense definition: every causal key is scored, non-selected ones get -inf,
    softmax with max subtraction, O = P V.  With q_pos0 > 0 the queries are a
    chunk of a longer sequence (positions q_pos0 .. q_pos0 + Nq - 1) over all
    N keys, with the selection of the whole sequence.
    """
    B, H, Nq, d = Q.shape
    Hkv, N = K.shape[1], K.shape[2]
    G = H // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.full((B, H, Nq, d), np.nan)
    LSE = np.full((B, H, Nq), np.nan)
    all_rows = np.arange(Nq) if rows is None else np.asarray(rows)
    for b in range(B):
        for h in range(H):
            g = h // G
            for c0 in range(0, all_rows.size, chunk):
                r = all_rows[c0:c0 + chunk]
                s, _ = _scores(Q[b, h], K[b, g], delta[b, h], evict[b, h], r, scale, gemm_dtype, q_pos0)
                m = s.max(axis=1, keepdims=True)
                p = np.exp(s - m)
                l = p.sum(axis=1, keepdims=True)
                O[b, h, r] = np.matmul(p / l, np.asarray(V[b, g], dtype=gemm_dtype)).astype(np.float64)
                LSE[b, h, r] = (m + np.log(l))[:, 0]
    return O, LSE


def attn_bwd(Q, K, V, delta, evict, dO, scale=None, gemm_dtype=np.float64, chunk: int = 1024):
    """Analytic backward of attn_fwd with the selection held constant.

    With P the masked softmax and L = sum(dO * O):
      dP = dO V^T,  D_t = sum_c dO_tc O_tc = sum_j P_tj dP_tj,
      dS = P * (dP - D),
      dQ = scale * dS K,   dK_g = scale * sum_{h in g} dS_h^T Q_h,
      dV_g = sum_{h in g} P_h^T dO_h,   ddelta_h = column sums of dS_h.
    Masked pairs have P = 0 hence dS = 0: zero gradient, as the section
    "Theoretical Guarantees for Safe Computation Skipping" states.
    Query rows are processed `chunk` at a time (sums over rows accumulate
    across chunks) so that large inputs fit in memory.

    Returns dQ [B,H,N,d], dK, dV [B,Hkv,N,d], ddelta [B,H,N], all float64.
    """
    B, H, N, d = Q.shape
    Hkv = K.shape[1]
    G = H // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = np.zeros((B, H, N, d))
    dK = np.zeros((B, Hkv, N, d))
    dV = np.zeros((B, Hkv, N, d))
    ddelta = np.zeros((B, H, N))
    f = lambda a: np.asarray(a, dtype=gemm_dtype)
    for b in range(B):
        for h in range(H):
            g = h // G
            Kg, Vg = f(K[b, g]), f(V[b, g])
            for c0 in range(0, N, chunk):
                rows = np.arange(c0, min(N, c0 + chunk))
                s, _ = _scores(Q[b, h], K[b, g], delta[b, h], evict[b, h], rows, scale, gemm_dtype)
                m = s.max(axis=1, keepdims=True)
                p = np.exp(s - m)
                P = p / p.sum(axis=1, keepdims=True)
                dP = np.matmul(f(dO[b, h, rows]), Vg.T).astype(np.float64)
                Dt = (P * dP).sum(axis=1, keepdims=True)
                dS = P * (dP - Dt)
                dQ[b, h, rows] = scale * np.matmul(f(dS), Kg).astype(np.float64)
                dK[b, g] += scale * np.matmul(f(dS).T, f(Q[b, h, rows])).astype(np.float64)
                dV[b, g] += np.matmul(f(P).T, f(dO[b, h, rows])).astype(np.float64)
                ddelta[b, h] += dS.sum(axis=0)
    return dQ, dK, dV, ddelta


# ----------------------------------------------------------------------------
# Gate backward (Delta and A are learnable; the method is end-to-end trainable)
# ----------------------------------------------------------------------------

def gate_bwd(V, Delta, A, ddelta, gemm_dtype=np.float64):
    """Gradients of sum(ddelta * delta) with delta = exp(A * softplus(v Delta)).

    d delta / d x = delta * A * sigmoid(x),  d delta / d A = delta * softplus(x).
    With gx = ddelta * delta * A * sigmoid(x):
      dA_h        = sum_{b,j} ddelta * delta * softplus(x),
      dDelta[r,h] = sum_{b,j} v_j[r] * gx[b,h,j],
      dV_gate[b,g,j,c] = sum_h gx[b,h,j] * Delta[g*d+c, h].
    The gate's share of dV is returned on its own (the caller adds it to the
    attention's dV).  Returns (dDelta [Hkv*d,H], dA [H], dV_gate [B,Hkv,N,d]).
    """
    B, Hkv, N, d = V.shape
    H = Delta.shape[1]
    x, delta = gate(V, Delta, A, gemm_dtype=gemm_dtype)
    dd = np.asarray(ddelta, dtype=np.float64)
    A64 = np.asarray(A, dtype=np.float64)
    gx = dd * delta * A64[None, :, None] * sigmoid(x)          # [B, H, N]
    dA = (dd * delta * softplus(x)).sum(axis=(0, 2))           # [H]
    v = np.asarray(V, dtype=np.float64).transpose(0, 2, 1, 3).reshape(B, N, Hkv * d)
    dDelta = np.einsum("bnr,bhn->rh", v, gx)
    dvf = np.einsum("bhn,rh->bnr", gx, np.asarray(Delta, dtype=np.float64))   # [B, N, Hkv*d]
    dV_gate = dvf.reshape(B, N, Hkv, d).transpose(0, 2, 1, 3).copy()
    return dDelta, dA, dV_gate


# ----------------------------------------------------------------------------
# Decode: one new query at position L-1 over an L-row cache
# ----------------------------------------------------------------------------

def decode_select(delta: np.ndarray, w: int) -> np.ndarray:
    """Keys selected for a query at position L-1 (all L keys are causal):
    the min(L, w) best under the selection order (delta descending, lower
    index first on ties).  Returns int64 [B, H, min(L, w)] sorted ascending by
    key index (the "Unified Training-Inference Architecture" section: the same
    selection at inference)."""
    B, H, L = delta.shape
    k = min(L, w)
    out = np.empty((B, H, k), dtype=np.int64)
    idx = np.arange(L)
    for b in range(B):
        for h in range(H):
            d = np.asarray(delta[b, h], dtype=np.float32).astype(np.float64)
            order = np.lexsort((idx, -d))       # primary -delta, secondary index
            out[b, h] = np.sort(order[:k])
    return out


def decode_select_append(prev_sel: np.ndarray, delta: np.ndarray, w: int) -> np.ndarray:
    """The decode selection after one key is appended to the cache, from the
    previous one (the "Unified Training-Inference Architecture" section: the
    same selection at every decode step; the m_t equation: the query at
    position t keeps the min(t+1, w) best keys of [0, t]).

    Because delta_j does not depend on the query, the best keys of [0, t] are
    the best of (the best keys of [0, t-1]) plus key t.  So with fewer than w
    keys selected the new key joins; otherwise it replaces the worst selected
    key (smallest delta; on equal delta the larger index, which loses the
    lower-index-first rule) exactly when it is better under the selection
    order.  The new key has the largest index, so that is when its delta is
    strictly larger.

    prev_sel [B, H, min(L-1, w)] ascending (the selection over the first L-1
    keys); delta [B, H, L].  Returns [B, H, min(L, w)] ascending, int64.
    """
    B, H, L = delta.shape
    kp = prev_sel.shape[2]
    assert kp == min(L - 1, w)
    k = min(L, w)
    out = np.empty((B, H, k), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            d = np.asarray(delta[b, h], dtype=np.float32)
            cur = [int(j) for j in prev_sel[b, h]]
            if kp < w:
                cur.append(L - 1)
            else:
                worst = cur[0]
                for j in cur[1:]:
                    if d[j] < d[worst] or (d[j] == d[worst] and j > worst):
                        worst = j
                if d[L - 1] > d[worst]:
                    cur.remove(worst)
                    cur.append(L - 1)
            out[b, h] = cur
    return out


def decode_attn(q, K, V, delta, sel, scale=None):
    """o = softmax(q k_j^T * scale + delta_j over the selected j) V.

    q [B, H, d] (or [B, H, 1, d]), K, V [B, Hkv, L, d], delta [B, H, L],
    sel [B, H, k] selected key indices.  Returns o [B, H, d], lse [B, H]."""
    q = np.asarray(q)
    if q.ndim == 4:
        q = q[:, :, 0, :]
    B, H, d = q.shape
    Hkv = K.shape[1]
    G = H // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = np.empty((B, H, d))
    lse = np.empty((B, H))
    for b in range(B):
        for h in range(H):
            g = h // G
            j = sel[b, h]
            kk = np.asarray(K[b, g, j], dtype=np.float64)
            vv = np.asarray(V[b, g, j], dtype=np.float64)
            s = kk @ np.asarray(q[b, h], dtype=np.float64) * scale + np.asarray(delta[b, h, j], dtype=np.float64)
            m = s.max()
            p = np.exp(s - m)
            l = p.sum()
            o[b, h] = (p / l) @ vv
            lse[b, h] = m + math.log(l)
    return o, lse


# ----------------------------------------------------------------------------
# Per-head windows ("Future Directions": adaptive window sizing; the window of
# each head is supplied, the pages give no rule for choosing it)
# ----------------------------------------------------------------------------

def head_windows(w_heads, w: int) -> np.ndarray:
    """The window each head selects with: w_heads[h] clamped to [1, w] (the
    largest window w bounds every head's)."""
    return np.clip(np.asarray(w_heads, dtype=np.int64), 1, w)


def topw_eviction_heads(delta: np.ndarray, w_heads, w: int) -> np.ndarray:
    """Eviction indices [B, H, N] when head h keeps the best min(t+1, W_h) keys
    of every prefix, W = head_windows(w_heads, w): the m_t equation applied to
    each head with its own window (the mask is per head, "a unique mask per
    attention head")."""
    B, H, N = delta.shape
    W = head_windows(w_heads, w)
    out = np.empty((B, H, N), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            out[b, h] = topw_eviction(delta[b, h], int(W[h]))
    return out


def decode_select_heads(delta: np.ndarray, w_heads, w: int) -> list:
    """Decode selection with per-head windows: a list over (b, h) in row-major
    order of the ascending selected keys of the query at position L-1 (row
    (b, h) holds min(L, W_h) keys)."""
    B, H, L = delta.shape
    W = head_windows(w_heads, w)
    return [decode_select(delta[b:b + 1, h:h + 1], int(W[h]))[0, 0] for b in range(B) for h in range(H)]


# ----------------------------------------------------------------------------
# Context-parallel prefill: the sequence split into contiguous shards, one per
# rank, with a single exchange of each shard's best keys
# ----------------------------------------------------------------------------
#
# The m_t equation selects, for a query at position t, the best min(t+1, W)
# keys of [0, t] by (delta desc, position asc).  The best keys of a union are
# among the best keys of its parts, so the best keys of the prefix [0, s_r) in
# front of shard r are among the best min(W, len_q) keys of every earlier shard
# q: each shard publishes those candidates once, and rank r rebuilds an exact
# stand-in for the prefix from the candidates of the shards before it.

def cp_candidates(delta, K, V, w_heads, w: int, shard_start: int):
    """The candidates a shard publishes: for every (b, h), the best
    min(W_h, len) keys of the shard by (delta desc, position asc), listed in
    ascending position, with their global position, delta and the K and V rows
    of head h's key/value head.  Entries past a row's count hold position -1,
    delta -inf and zero rows.

    delta [B, H, len], K, V [B, Hkv, len, d] (the shard's part).  Returns a dict
    pos [B, H, w] int64, delta [B, H, w] float32, K, V [B, H, w, d]."""
    B, H, L = delta.shape
    Hkv, d = K.shape[1], K.shape[3]
    G = H // Hkv
    W = head_windows(np.full(H, w) if w_heads is None else w_heads, w)
    pos = np.full((B, H, w), -1, dtype=np.int64)
    dl = np.full((B, H, w), -np.inf, dtype=np.float32)
    Kc = np.zeros((B, H, w, d), dtype=K.dtype)
    Vc = np.zeros((B, H, w, d), dtype=V.dtype)
    for b in range(B):
        for h in range(H):
            sel = decode_select(delta[b:b + 1, h:h + 1], int(W[h]))[0, 0]   # ascending shard positions
            k = sel.size
            pos[b, h, :k] = shard_start + sel
            dl[b, h, :k] = np.asarray(delta[b, h, sel], dtype=np.float32)
            Kc[b, h, :k] = K[b, h // G, sel]
            Vc[b, h, :k] = V[b, h // G, sel]
    return {"pos": pos, "delta": dl, "K": Kc, "V": Vc}


def cp_prefix_len(G: int, w: int, prefix_len: int) -> int:
    """Rows that stand in for the prefix of a shard: min(G w, prefix_len)."""
    return min(G * w, prefix_len)


def cp_compact(cands, prefix_len: int, delta, K, V, w_heads, w: int):
    """The compacted sequence rank r attends over: a stand-in for the prefix
    [0, prefix_len) followed by the shard's own keys.

    cands: the cp_candidates of every earlier shard, in shard order.  For each
    (b, h) the best min(W_h, prefix_len) of the merged candidates (delta desc,
    position asc) are the best keys of the whole prefix.  For each (b, g) the
    stand-in holds the union of those sets over the heads of group g, ascending
    in position, after P - |union| padding rows (P = cp_prefix_len): padding
    rows have zero K and V and delta -inf for every head; a union key that head
    h did not select has delta -inf for head h.  Then the shard's own keys.

    Returns (K_c, V_c [B, Hkv, P + len, d], delta_c [B, H, P + len], P,
    pos_c [B, Hkv, P + len]: the original position of every row, -1 for padding)."""
    B, H, L = delta.shape
    Hkv, d = K.shape[1], K.shape[3]
    G = H // Hkv
    W = head_windows(np.full(H, w) if w_heads is None else w_heads, w)
    P = cp_prefix_len(G, w, prefix_len)
    Kc = np.zeros((B, Hkv, P + L, d), dtype=K.dtype)
    Vc = np.zeros((B, Hkv, P + L, d), dtype=V.dtype)
    dc = np.full((B, H, P + L), -np.inf, dtype=np.float32)
    Kc[:, :, P:] = K
    Vc[:, :, P:] = V
    dc[:, :, P:] = delta
    pc = np.full((B, Hkv, P + L), -1, dtype=np.int64)
    pc[:, :, P:] = prefix_len + np.arange(L)
    for b in range(B):
        for g in range(Hkv):
            chosen = {}     # position -> (K row, V row, {head: delta})
            for hh in range(G):
                h = g * G + hh
                pos = np.concatenate([c["pos"][b, h] for c in cands]) if cands else np.zeros(0, np.int64)
                dl = np.concatenate([c["delta"][b, h] for c in cands]) if cands else np.zeros(0, np.float32)
                kr = np.concatenate([c["K"][b, h] for c in cands]) if cands else np.zeros((0, d))
                vr = np.concatenate([c["V"][b, h] for c in cands]) if cands else np.zeros((0, d))
                real = np.nonzero(pos >= 0)[0]
                order = sorted(real, key=lambda i: (-float(dl[i]), int(pos[i])))
                for i in order[:min(int(W[h]), prefix_len)]:
                    ent = chosen.setdefault(int(pos[i]), (kr[i], vr[i], {}))
                    ent[2][h] = dl[i]
            keys = sorted(chosen)
            assert len(keys) <= P
            base = P - len(keys)
            for n, j in enumerate(keys):
                kr, vr, dh = chosen[j]
                Kc[b, g, base + n] = kr
                Vc[b, g, base + n] = vr
                pc[b, g, base + n] = j
                for h, v in dh.items():
                    dc[b, h, base + n] = v
    return Kc, Vc, dc, P, pc


def cp_shard_bounds(N: int, R: int):
    """Contiguous shards of [0, N) for R ranks: shard r = [r n, min((r+1) n, N)), n = ceil(N / R)."""
    n = -(-N // R)
    return [(min(r * n, N), min((r + 1) * n, N)) for r in range(R)]
