"""Context-parallel prefill: the sequence split into contiguous shards, one per
rank (one GPU each), with a single exchange of each shard's best keys.

The m_t equation of "Trainable Dynamic Mask Sparse Attention" (section
"Dynamic Sparse Mask Generation") keeps, for a query at position t, the best
min(t+1, w) keys of [0, t] by delta.  The best keys of a union are among the
best keys of its parts, so rank r needs from the ranks before it only their
best keys (dma_cp_candidates), from which it rebuilds an exact stand-in for the
prefix in front of its shard (dma_cp_compact), and then runs the ordinary
selection and attention on that compacted sequence as a chunk of queries.

Every step of the computation runs in libdma's kernels; this module allocates
with torch and moves the fixed-size candidate buffers between ranks with
torch.distributed (an all-gather: NCCL between GPUs, gloo between host
processes).
"""
from __future__ import annotations

from . import alloc_workspace, attn_fwd, cp_candidates, cp_compact, cp_layout, gate, make_params, topk_mask

__all__ = ["shard_bounds", "exchange", "candidates", "compact_and_attend", "prefill_forward"]


def shard_bounds(N: int, world: int):
    """Contiguous shards of [0, N) in rank order: ceil(N / world) positions each (the last may be shorter)."""
    n = -(-N // world)
    return [(min(r * n, N), min((r + 1) * n, N)) for r in range(world)]


def exchange(cand, group=None):
    """All-gather of every rank's candidate buffer (a 1-D uint8 tensor of the same size on every
    rank): returns [world, nbytes], row q = rank q's buffer.  Every rank takes part, in the same order."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    outs = [torch.empty_like(cand) for _ in range(world)]
    dist.all_gather(outs, cand, group=group)
    return torch.stack(outs)


def candidates(p_shard, shard_start, delta, K, V, stream=None):
    """The shard's candidate buffer (a uint8 tensor of cand_bytes) for shard problem p_shard starting
    at global position shard_start."""
    import torch
    lay = cp_layout(p_shard, 0, 0)
    ws = torch.zeros(lay.ws_bytes, dtype=torch.uint8, device=K.device)
    cand = torch.empty(lay.cand_bytes, dtype=torch.uint8, device=K.device)
    cp_candidates(p_shard, shard_start, delta, K, V, cand, ws, stream)
    return cand


def compact_and_attend(p_shard, shard_start, prev, Q, K, V, delta, stream=None):
    """From the candidate buffers of the shards before this one (prev: [n_prev, cand_bytes] uint8,
    or None for the first shard), the compacted sequence and the attention of the shard's queries
    over it.  Returns a dict with O [B, H, len, d], LSE [B, H, len] and the compacted Kc, Vc,
    delta_c, pos_c and evict (its selection)."""
    import torch
    n_prev = 0 if prev is None else int(prev.shape[0])
    lay = cp_layout(p_shard, shard_start, n_prev)
    B, H, Hkv, n, d = p_shard.B, p_shard.H, p_shard.Hkv, p_shard.N, p_shard.d
    P = lay.prefix_rows
    Nc = P + n
    dev = K.device
    ws = torch.zeros(lay.ws_bytes, dtype=torch.uint8, device=dev)
    delta_c = torch.empty((B, H, Nc), dtype=torch.float32, device=dev)
    Kc = torch.empty((B, Hkv, Nc, d), dtype=K.dtype, device=dev)
    Vc = torch.empty((B, Hkv, Nc, d), dtype=V.dtype, device=dev)
    pos_c = torch.empty((B, Hkv, Nc), dtype=torch.int32, device=dev)
    cands = None if prev is None else prev.contiguous()
    cp_compact(p_shard, shard_start, n_prev, cands, delta, K, V, delta_c, Kc, Vc, pos_c, ws, stream)
    w_heads = p_shard.w_heads
    p2 = make_params(B, H, Hkv, Nc, d, p_shard.w, Nq=n, dtype=p_shard.dtype, w_heads=w_heads, forward_only=True)
    ws2 = alloc_workspace(p2, dev, stream)
    evict = torch.empty((B, H, Nc), dtype=torch.int32, device=dev)
    O = torch.empty((B, H, n, d), dtype=Q.dtype, device=dev)
    LSE = torch.empty((B, H, n), dtype=torch.float32, device=dev)
    topk_mask(p2, delta_c, evict, ws2, stream)
    attn_fwd(p2, Q, Kc, Vc, delta_c, evict, ws2, O, LSE, stream)
    return {"O": O, "LSE": LSE, "Kc": Kc, "Vc": Vc, "delta_c": delta_c, "pos_c": pos_c, "evict": evict,
            "prefix_rows": P, "status_word": ws[lay.off_status: lay.off_status + 4]}


def prefill_forward(p_shard, shard_start, Q, K, V, Delta, A, rank, group=None):
    """This rank's part of a context-parallel prefill forward: gate on the shard, candidates, the
    exchange, compaction and attention, all on torch's current stream (the one the collective runs
    on).  p_shard: the problem of this rank's shard (N = its length;
    the other fields those of the whole sequence); Q, K, V: the shard's rows.  Every rank of the
    group calls it once with its own shard (the exchange is collective).  Returns the dict of
    compact_and_attend plus the shard's delta."""
    import torch
    B, H, n = p_shard.B, p_shard.H, p_shard.N
    delta = torch.empty((B, H, n), dtype=torch.float32, device=K.device)
    gate(p_shard, V, Delta, A, delta, None, None)
    cand = candidates(p_shard, shard_start, delta, K, V)
    allc = exchange(cand, group)
    prev = allc[:rank] if rank > 0 else None
    out = compact_and_attend(p_shard, shard_start, prev, Q, K, V, delta)
    out["delta"] = delta
    return out
