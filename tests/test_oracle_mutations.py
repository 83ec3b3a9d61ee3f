"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in the oracle (on the CPU, through monkeypatch)
and checks that at least one pin then fails: a dropped term of softplus, the
tie rule reversed, the scale applied to delta as well, a transposed Delta, a
missing row-max subtraction sign, a wrong sign in the backward, and the two tie
mistakes of the decode append rule (an equal new key entering; the smaller
index leaving among equal worst keys).
"""
import math

import numpy as np
import pytest

import oracle
import oracle.dma_oracle as od
import test_oracle_attn as TA
import test_oracle_gate as TG
import test_oracle_topw as TT


def _fails(fn, *a, **k):
    try:
        fn(*a, **k)
    except (AssertionError, ValueError):
        return True
    return False


def test_softplus_without_log1p_term_is_caught(monkeypatch):
    monkeypatch.setattr(od, "softplus", lambda x: np.maximum(np.asarray(x, dtype=np.float64), 0.0))
    assert _fails(TG.test_zero_delta_weights_give_two_to_the_A)


def test_channel_major_concatenation_is_caught(monkeypatch):
    def bad_gate(V, Delta, A, gemm_dtype=np.float64):
        B, Hkv, N, d = V.shape
        # v_j[c*Hkv + g] instead of v_j[g*d + c]
        v = np.asarray(V, dtype=np.float64).transpose(0, 2, 3, 1).reshape(B, N, Hkv * d)
        x = np.matmul(v, np.asarray(Delta, dtype=np.float64)).transpose(0, 2, 1).copy()
        return x, np.exp(np.asarray(A)[None, :, None] * od.softplus(x))

    monkeypatch.setattr(oracle, "gate", bad_gate)
    assert _fails(TG.test_head_concatenation_and_index_roles)


def test_reversed_tie_rule_is_caught(monkeypatch):
    import heapq

    def bad(delta_row, w):
        d = np.asarray(delta_row, dtype=np.float32)
        N = d.shape[0]
        e = np.full(N, N, dtype=np.int64)
        heap = []
        for t in range(N):
            heapq.heappush(heap, (float(d[t]), t))   # ties: higher index wins
            if len(heap) > w:
                _, j = heapq.heappop(heap)
                e[j] = t
        return e

    monkeypatch.setattr(oracle, "topw_eviction", bad)
    assert _fails(TT.test_worked_example_by_hand)


def test_scaling_delta_too_is_caught(monkeypatch):
    real = od._scores

    def bad(Qh, Kg, delta_h, e_h, rows, scale, gemm_dtype, q_pos0=0):
        return real(Qh, Kg, np.asarray(delta_h) * scale, e_h, rows, scale, gemm_dtype, q_pos0)

    monkeypatch.setattr(od, "_scores", bad)
    assert _fails(TA.test_full_window_is_dense_causal_attention_with_bias)


def test_off_by_one_causal_mask_is_caught(monkeypatch):
    def bad_mask(e, q_rows=None):
        N = e.shape[-1]
        t = np.arange(N) if q_rows is None else np.asarray(q_rows)
        j = np.arange(N)
        return (j[None, :] < t[:, None]) & (t[:, None] < e[None, :])

    monkeypatch.setattr(oracle, "mask_from_eviction", bad_mask)
    assert _fails(TT.test_eviction_pass_equals_brute_force, "uniform", 0, 17, 4)


def test_wrong_sign_in_backward_is_caught(monkeypatch):
    real = od.attn_bwd

    def bad(*a, **k):
        dQ, dK, dV, dd = real(*a, **k)
        return dQ, -dK, dV, dd

    monkeypatch.setattr(oracle, "attn_bwd", bad)
    assert _fails(TA.test_backward_matches_central_differences, 3)


def test_gate_backward_missing_sigmoid_is_caught(monkeypatch):
    monkeypatch.setattr(od, "sigmoid", lambda x: np.ones_like(np.asarray(x, dtype=np.float64)))
    assert _fails(TA.test_gate_backward_matches_central_differences)


def _append_with(ge: bool, smaller_index_is_worst: bool):
    def bad(prev_sel, delta, w):
        B, H, L = delta.shape
        out = []
        for b in range(B):
            rows = []
            for h in range(H):
                d = np.asarray(delta[b, h], dtype=np.float32)
                cur = [int(j) for j in prev_sel[b, h]]
                if len(cur) < w:
                    cur.append(L - 1)
                else:
                    worst = cur[0]
                    for j in cur[1:]:
                        tie_pick = j < worst if smaller_index_is_worst else j > worst
                        if d[j] < d[worst] or (d[j] == d[worst] and tie_pick):
                            worst = j
                    if (d[L - 1] >= d[worst]) if ge else (d[L - 1] > d[worst]):
                        cur.remove(worst)
                        cur.append(L - 1)
                rows.append(sorted(cur))
            out.append(rows)
        return np.array(out, dtype=np.int64)
    return bad


@pytest.mark.parametrize("ge, smaller", [(True, False), (False, True)])
def test_append_tie_mistakes_are_caught(monkeypatch, ge, smaller):
    # a new key that only equals the worst one must not enter; among equal worst values the larger
    # index leaves
    monkeypatch.setattr(oracle, "decode_select_append", _append_with(ge, smaller))
    assert _fails(TA.test_decode_select_append_equals_the_full_selection_at_every_length) or \
        _fails(TA.test_decode_select_append_cases)


def test_candidates_of_the_previous_shard_only_are_caught(monkeypatch):
    """A sharded prefill that merges only the shard just before instead of every earlier one."""
    import test_oracle_cp as TC
    real = od.cp_compact

    def bad(cands, prefix_len, *a, **k):
        return real(cands[-1:], prefix_len, *a, **k)

    monkeypatch.setattr(oracle, "cp_compact", bad)
    assert _fails(TC.test_sharded_equals_whole_sequence, 3, 37, None)


def test_prefix_stand_in_of_one_window_is_caught(monkeypatch):
    """A stand-in of w rows for the prefix (one head's window) instead of G w: the union of the
    group's heads does not fit."""
    import test_oracle_cp as TC
    monkeypatch.setattr(oracle, "cp_prefix_len", lambda G, w, prefix_len: min(w, prefix_len))
    monkeypatch.setattr(od, "cp_prefix_len", lambda G, w, prefix_len: min(w, prefix_len))
    assert _fails(TC.test_sharded_equals_whole_sequence, 2, 37, None)
