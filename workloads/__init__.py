"""Seeded synthetic inputs for the Dynamic Mask Attention hot path.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark.  It only draws random numbers and rounds them to the storage type;
it contains none of the method's arithmetic (no gate, no selection, no
attention), so neither side of a parity check borrows anything from the other
through it.

Workload shapes follow the five configurations the method is measured on
(tiny, prefill, long, decode, train).  Draw order for every workload is fixed:
Q, K, V, Delta, A, scaled key positions, dO.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "get",
    "bf16_round",
    "bf16_bits_to_f32",
    "make_inputs",
    "make_delta",
]


@dataclass(frozen=True)
class Workload:
    """Shape and seed of one synthetic workload.

    B batch, H query heads, Hkv key/value heads (H % Hkv == 0), N key length
    (sequence length; for decode the cache length), Nq query rows (N for
    prefill/train, 1 for decode), d head dim, w window of the top-w selection.
    dtype is the storage type of Q, K, V, Delta and dO ("f32" or "bf16").
    scaled_frac is the fraction of key positions whose K and V rows are
    multiplied by 4 (exact in bf16) to skew the gate.
    """

    name: str
    B: int
    H: int
    Hkv: int
    N: int
    d: int
    w: int
    dtype: str
    seed: int
    Nq: int = -1
    scaled_frac: float = 0.0
    with_dO: bool = False

    def __post_init__(self):
        if self.Nq == -1:
            object.__setattr__(self, "Nq", self.N)
        assert self.H % self.Hkv == 0

    @property
    def G(self) -> int:
        return self.H // self.Hkv

    @property
    def q_pos0(self) -> int:
        return self.N - self.Nq

    def kept_pairs(self) -> int:
        """Sum over query rows of min(t+1, w) per (b, h): the number of
        (query, key) pairs the mask keeps.  It does not depend on delta."""
        t = np.arange(self.q_pos0, self.N, dtype=np.int64)
        return int(np.minimum(t + 1, self.w).sum()) * self.B * self.H

    def with_(self, **kw) -> "Workload":
        """A copy with some fields changed.  Changing N keeps the query-row
        mode: prefill/train (Nq == N) follows the new N, decode keeps Nq = 1."""
        if "N" in kw and "Nq" not in kw:
            kw["Nq"] = 1 if self.Nq == 1 and self.N > 1 else kw["N"]
        return replace(self, **kw)


WORKLOADS = {
    # B=1, H=2 sharing one KV head, N=256, d=64, w=64; fp32 inputs; seed 0.
    "tiny": Workload("tiny", B=1, H=2, Hkv=1, N=256, d=64, w=64, dtype="f32", seed=0),
    # GQA prefill: B=1, H=16, Hkv=8, N=4096, d=128, w=1024, bf16; seed 1.
    "prefill": Workload("prefill", B=1, H=16, Hkv=8, N=4096, d=128, w=1024, dtype="bf16", seed=1),
    # Long prefill with 5% of key positions scaled by 4; seed 2.
    "long": Workload("long", B=1, H=32, Hkv=8, N=16384, d=128, w=2048, dtype="bf16", seed=2,
                     scaled_frac=0.05),
    # Decode: 8 sequences, one new query each over a 65536-row cache; seed 3.
    "decode": Workload("decode", B=8, H=32, Hkv=8, N=65536, d=128, w=2048, dtype="bf16", seed=3,
                       Nq=1),
    # Training step fwd+bwd with dO; seed 4.
    "train": Workload("train", B=2, H=16, Hkv=8, N=8192, d=128, w=2048, dtype="bf16", seed=4,
                      with_dO=True),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def bf16_round(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round float32 values to bfloat16 with round-to-nearest-even.

    Returns (values as float32, raw bf16 bits as uint16).  The float32 array
    holds exactly the bf16 values, so the same numbers reach both the GPU
    (as bits) and the oracle (as floats).  Inputs are finite draws.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32), (r >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bits (uint16) to float32 exactly."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Inputs:
    """Seeded inputs of one workload.

    Float arrays hold the exact stored values (bf16-representable when
    dtype == "bf16").  `bits` maps a name to its uint16 bf16 bit pattern for
    the bf16 tensors (what the GPU receives).
    """

    Q: np.ndarray       # [B, H, Nq, d]
    K: np.ndarray       # [B, Hkv, N, d]
    V: np.ndarray       # [B, Hkv, N, d]
    Delta: np.ndarray   # [Hkv*d, H]
    A: np.ndarray       # [H] float32
    scaled_pos: np.ndarray  # int64 positions whose K, V rows were scaled by 4
    dO: np.ndarray | None   # [B, H, Nq, d] or None
    bits: dict


def _normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def make_inputs(wl: Workload, with_dO: bool | None = None, bf16_values: bool = False) -> Inputs:
    """Draw the inputs of `wl` from numpy's default_rng(seed) in the fixed
    order Q, K, V, Delta, A, scaled positions, dO.

    bf16_values: for dtype "f32", round Q, K, V, Delta and dO to
    bf16-representable values (still stored as float32)."""
    if with_dO is None:
        with_dO = wl.with_dO
    rng = np.random.default_rng(wl.seed)
    B, H, Hkv, N, Nq, d = wl.B, wl.H, wl.Hkv, wl.N, wl.Nq, wl.d
    Q = _normal(rng, (B, H, Nq, d))
    K = _normal(rng, (B, Hkv, N, d))
    V = _normal(rng, (B, Hkv, N, d))
    Delta = _normal(rng, (Hkv * d, H), std=0.02)
    A = rng.uniform(-1.0, 0.0, size=H).astype(np.float32)
    n_scaled = int(round(wl.scaled_frac * N))
    if n_scaled > 0:
        pos = np.sort(rng.choice(N, size=n_scaled, replace=False)).astype(np.int64)
        K[:, :, pos, :] *= np.float32(4.0)
        V[:, :, pos, :] *= np.float32(4.0)
    else:
        pos = np.zeros(0, dtype=np.int64)
    dO = _normal(rng, (B, H, Nq, d)) if with_dO else None
    bits = {}
    if wl.dtype == "bf16":
        Q, bits["Q"] = bf16_round(Q)
        K, bits["K"] = bf16_round(K)
        V, bits["V"] = bf16_round(V)
        Delta, bits["Delta"] = bf16_round(Delta)
        if dO is not None:
            dO, bits["dO"] = bf16_round(dO)
    elif wl.dtype == "f32":
        if bf16_values:
            Q, K, V, Delta = (bf16_round(a)[0] for a in (Q, K, V, Delta))
            if dO is not None:
                dO = bf16_round(dO)[0]
    else:
        raise ValueError(f"unknown dtype {wl.dtype}")
    return Inputs(Q=Q, K=K, V=V, Delta=Delta, A=A, scaled_pos=pos, dO=dO, bits=bits)


def make_delta(shape, seed: int, kind: str = "uniform", levels: int = 0) -> np.ndarray:
    """Synthetic gate values for exercising the selection on its own.

    kind: "uniform"   float32 draws in (0, 1];
          "levels"    draws from `levels` distinct values (many exact ties);
          "increasing" strictly increasing along the last axis;
          "decreasing" strictly decreasing along the last axis;
          "constant"  every value equal (all ties).
    """
    rng = np.random.default_rng(seed)
    shape = tuple(shape)
    n = shape[-1]
    if kind == "uniform":
        x = 1.0 - rng.random(size=shape, dtype=np.float32)  # (0, 1]
    elif kind == "levels":
        assert levels >= 1
        vals = np.sort(1.0 - rng.random(size=levels, dtype=np.float32))
        x = vals[rng.integers(0, levels, size=shape)]
    elif kind == "increasing":
        base = (np.arange(n, dtype=np.float32) + 1.0) / np.float32(n + 1)
        x = np.broadcast_to(base, shape).copy()
    elif kind == "decreasing":
        base = (np.arange(n, 0, -1, dtype=np.float32)) / np.float32(n + 1)
        x = np.broadcast_to(base, shape).copy()
    elif kind == "constant":
        x = np.full(shape, 0.5, dtype=np.float32)
    else:
        raise ValueError(kind)
    return np.ascontiguousarray(x, dtype=np.float32)
