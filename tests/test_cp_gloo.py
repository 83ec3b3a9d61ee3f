"""Context-parallel prefill across two host processes (gloo, world_size 2): each
rank holds one shard, publishes its candidates through the library's exchange
plumbing (trainable_dynamic_mask_b200.cp.exchange, the all-gather the GPU path
uses over NCCL), rebuilds the prefix stand-in from the ranks before it and
computes its queries' attention.  The computation on each rank is the oracle's
(this test runs without a GPU); the result must equal the whole-sequence
oracle's rows of that shard."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _pack(c):
    parts = [c["pos"].astype(np.int32), c["delta"].astype(np.float32), c["K"].astype(np.float32),
             c["V"].astype(np.float32)]
    return torch.from_numpy(np.concatenate([np.ascontiguousarray(a).view(np.uint8).ravel() for a in parts]))


def _unpack(buf, B, H, w, d):
    b = buf.numpy()
    out, off = {}, 0
    for name, dt, shape in (("pos", np.int32, (B, H, w)), ("delta", np.float32, (B, H, w)),
                            ("K", np.float32, (B, H, w, d)), ("V", np.float32, (B, H, w, d))):
        n = int(np.prod(shape)) * 4
        out[name] = b[off: off + n].view(dt).reshape(shape)
        off += n
    out["pos"] = out["pos"].astype(np.int64)
    return out


def _rank_main(rank, world, port, cfg, out):
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle
    from trainable_dynamic_mask_b200 import cp
    from workloads import get, make_inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=120))
    try:
        wl = get("tiny").with_(**cfg)
        I = make_inputs(wl)                       # every rank draws the same seeded inputs ...
        _, d = oracle.gate(I.V, I.Delta, I.A)
        d32 = d.astype(np.float32)
        s0, s1 = cp.shard_bounds(wl.N, world)[rank]   # ... and uses only its shard for the computation
        c = oracle.cp_candidates(d32[:, :, s0:s1], I.K[:, :, s0:s1], I.V[:, :, s0:s1], None, wl.w, s0)
        allc = cp.exchange(_pack(c))
        prev = [_unpack(allc[q], wl.B, wl.H, wl.w, wl.d) for q in range(rank)]
        Kc, Vc, dc, P, pc = oracle.cp_compact(prev, s0, d32[:, :, s0:s1], I.K[:, :, s0:s1], I.V[:, :, s0:s1],
                                              None, wl.w)
        ec = oracle.topw_eviction_heads(dc, np.full(wl.H, wl.w), wl.w)
        O, L = oracle.attn_fwd(I.Q[:, :, s0:s1], Kc, Vc, dc.astype(np.float64), ec, q_pos0=P)
        # the check: the whole sequence, computed by this rank alone
        e = oracle.topw_eviction_heads(d32, np.full(wl.H, wl.w), wl.w)
        O_f, L_f = oracle.attn_fwd(I.Q, I.K, I.V, d32.astype(np.float64), e, rows=np.arange(s0, s1))
        out[rank] = (float(np.abs(O - O_f[:, :, s0:s1]).max()), float(np.abs(L - L_f[:, :, s0:s1]).max()), P,
                     int(allc.shape[0]))
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("cfg", [dict(B=2, H=4, Hkv=2, N=700, d=16, w=90, seed=5),
                                 dict(B=1, H=2, Hkv=1, N=300, d=8, w=500, seed=6)],
                         ids=["window_below_shard", "window_above_sequence"])
def test_two_ranks_equal_whole_sequence(cfg):
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), cfg, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank, (eo, el, P, n) in res.items():
        assert n == world
        assert eo < 1e-12 and el < 1e-12, (rank, eo, el)
    assert res[0][2] == 0
