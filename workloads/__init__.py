"""Seeded synthetic inputs for the heterogeneous-batch LoRA branch.

This module only draws random numbers and lays them out.  It holds none of the
method's arithmetic (no contraction, no scaling, no grouping): the CUDA path and
the fp64 oracle both consume what it produces, and neither is imported here.

The five workloads follow the shapes named for this method's benchmark:

  1. tiny          d_in=d_out=256, 4 slots of rank 8 (alpha 16), 32 rows in
                   segments of lengths [8,4,6,9,5] on slots [0,-1,1,2,3].
  2. qproj_decode  Llama-3-8B q_proj, d_in=d_out=4096, 64 slots of rank 16
                   (alpha 32), 256 decode rows, slots Zipf(1.1), 10% base-only,
                   rows in arrival order.
  3. qkv_prefill   fused QKV, d_in=4096, d_out=6144, 8 requests with lengths
                   uniform in [128, 2048], each on its own rank-64 slot (alpha 128).
  4. mixed_mlp     1024 slots, ranks uniform in {8,16,32,64}, alpha = 2r;
                   512 decode rows (Zipf 1.1) + 4 prefill requests of 512 rows;
                   projections gate/up 4096->14336 and down 14336->4096.
  5. block70b      d=8192, 128 slots of rank 16 (alpha 32), 2048 decode rows
                   (Zipf 1.1), 5% base-only; projections q, k, v, o, gate, up, down.

Distributions: adapter weights N(0, 0.02), activations X and base outputs Y0
N(0, 1), all drawn as float32 by numpy's PCG64 ``default_rng`` and rounded to
bfloat16 with round-to-nearest-even.  Arrays of bf16 values are returned as
``uint16`` bit patterns.

Recipe (per workload seed):
  * ``rng = default_rng(seed)`` draws, in this order: slot ranks (workload 4
    only), the per-row slot map, the base-only mask, request lengths
    (workload 3 only).
  * each projection ``j`` (0-based, in the listed order) draws from
    ``default_rng([seed, j + 1])``: A then B for every referenced slot in
    ascending slot order, then X, then Y0.
  * the base weight W of projection ``j`` (used where the base GEMM itself is part
    of the computation) comes from ``default_rng([seed, j + 1, 87])``.

``scale_rows`` shrinks the row counts (same structure, fewer rows) so the oracle
finishes in seconds; full-size workloads are used for sampled parity checks and
for the benchmark.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

WEIGHT_STD = 0.02
RANK_BUCKETS = (8, 16, 32, 64)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the 16-bit patterns as ``uint16``.  Inputs here are finite normals,
    so no NaN handling is needed; an infinity stays an infinity.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


def _zipf_slots(rng: np.random.Generator, n_slots: int, n: int, s: float = 1.1) -> np.ndarray:
    """Bounded Zipf over slots: P(slot = k-1) proportional to k^-s, k = 1..n_slots."""
    k = np.arange(1, n_slots + 1, dtype=np.float64)
    p = k ** (-s)
    p /= p.sum()
    return rng.choice(n_slots, size=n, p=p).astype(np.int32)


@dataclass
class Projection:
    """One linear layer's LoRA inputs: adapters for the referenced slots, X and Y0."""
    name: str
    d_in: int
    d_out: int
    A: Dict[int, np.ndarray]   # slot -> uint16 [rank, d_in]  (PEFT layout)
    B: Dict[int, np.ndarray]   # slot -> uint16 [d_out, rank]
    X: np.ndarray              # uint16 [n_rows, d_in]
    Y0: np.ndarray             # uint16 [n_rows, d_out]


@dataclass
class Workload:
    name: str
    seed: int
    n_slots: int
    r_max: int
    slot_rank: np.ndarray          # int32 [n_slots]
    slot_alpha: np.ndarray         # float64 [n_slots]
    row_slot: np.ndarray           # int32 [n_rows]; -1 = base only
    proj_shapes: List[tuple]       # (name, d_in, d_out)
    phase: str                     # "decode", "prefill" or "mixed"
    _proj_cache: Dict[int, Projection] = field(default_factory=dict, repr=False)

    @property
    def n_rows(self) -> int:
        return int(self.row_slot.shape[0])

    @property
    def referenced_slots(self) -> np.ndarray:
        s = np.unique(self.row_slot)
        return s[s >= 0].astype(np.int32)

    def projection(self, j: int, cache: bool = False) -> Projection:
        """Draw projection ``j`` (deterministic in (seed, j))."""
        if j in self._proj_cache:
            return self._proj_cache[j]
        name, d_in, d_out = self.proj_shapes[j]
        rng = np.random.default_rng([self.seed, j + 1])
        A: Dict[int, np.ndarray] = {}
        B: Dict[int, np.ndarray] = {}
        for s in self.referenced_slots.tolist():
            r = int(self.slot_rank[s])
            A[s] = _normal_bf16(rng, (r, d_in), WEIGHT_STD)
            B[s] = _normal_bf16(rng, (d_out, r), WEIGHT_STD)
        X = _normal_bf16(rng, (self.n_rows, d_in), 1.0)
        Y0 = _normal_bf16(rng, (self.n_rows, d_out), 1.0)
        p = Projection(name, d_in, d_out, A, B, X, Y0)
        if cache:
            self._proj_cache[j] = p
        return p

    def base_weight(self, j: int) -> np.ndarray:
        """Base weight W [d_out, d_in] of projection ``j`` (nn.Linear layout), bf16 bits
        drawn N(0, 0.02) from its own stream ``default_rng([seed, j + 1, 87])``, so that
        the projection's other draws do not depend on whether it is made."""
        _, d_in, d_out = self.proj_shapes[j]
        return _normal_bf16(np.random.default_rng([self.seed, j + 1, 87]), (d_out, d_in), WEIGHT_STD)

    def projections(self):
        for j in range(len(self.proj_shapes)):
            yield self.projection(j)


def _base_mask(rng: np.random.Generator, row_slot: np.ndarray, frac: float) -> np.ndarray:
    n = row_slot.shape[0]
    m = int(round(frac * n))
    if m > 0:
        idx = rng.choice(n, size=m, replace=False)
        row_slot = row_slot.copy()
        row_slot[idx] = -1
    return row_slot


def tiny(seed: int = 0) -> Workload:
    lengths = [8, 4, 6, 9, 5]
    slots = [0, -1, 1, 2, 3]
    row_slot = np.concatenate([np.full(l, s, np.int32) for l, s in zip(lengths, slots)])
    return Workload("tiny", seed, 4, 8, np.full(4, 8, np.int32), np.full(4, 16.0),
                    row_slot, [("proj", 256, 256)], "mixed")


def qproj_decode(seed: int = 1, n_rows: int = 256) -> Workload:
    rng = np.random.default_rng(seed)
    n_slots = 64
    row_slot = _zipf_slots(rng, n_slots, n_rows)
    row_slot = _base_mask(rng, row_slot, 0.10)
    return Workload("qproj_decode", seed, n_slots, 16, np.full(n_slots, 16, np.int32),
                    np.full(n_slots, 32.0), row_slot, [("q_proj", 4096, 4096)], "decode")


def qkv_prefill(seed: int = 2, lo: int = 128, hi: int = 2048) -> Workload:
    rng = np.random.default_rng(seed)
    n_req = 8
    lengths = rng.integers(lo, hi, size=n_req, endpoint=True)
    slots = rng.permutation(n_req).astype(np.int32)
    row_slot = np.concatenate([np.full(int(l), s, np.int32) for l, s in zip(lengths, slots)])
    return Workload("qkv_prefill", seed, n_req, 64, np.full(n_req, 64, np.int32),
                    np.full(n_req, 128.0), row_slot, [("qkv_proj", 4096, 6144)], "prefill")


def mixed_mlp(seed: int = 3, n_decode: int = 512, prefill_len: int = 512,
              n_prefill: int = 4) -> Workload:
    rng = np.random.default_rng(seed)
    n_slots = 1024
    ranks = rng.choice(np.array(RANK_BUCKETS, np.int32), size=n_slots).astype(np.int32)
    decode = _zipf_slots(rng, n_slots, n_decode)
    prefill_slots = _zipf_slots(rng, n_slots, n_prefill)
    parts = [decode] + [np.full(prefill_len, s, np.int32) for s in prefill_slots.tolist()]
    row_slot = np.concatenate(parts).astype(np.int32)
    return Workload("mixed_mlp", seed, n_slots, 64, ranks, 2.0 * ranks.astype(np.float64),
                    row_slot,
                    [("gate_proj", 4096, 14336), ("up_proj", 4096, 14336),
                     ("down_proj", 14336, 4096)], "mixed")


def block70b(seed: int = 4, n_rows: int = 2048) -> Workload:
    rng = np.random.default_rng(seed)
    n_slots = 128
    row_slot = _zipf_slots(rng, n_slots, n_rows)
    row_slot = _base_mask(rng, row_slot, 0.05)
    d = 8192
    return Workload("block70b", seed, n_slots, 16, np.full(n_slots, 16, np.int32),
                    np.full(n_slots, 32.0), row_slot,
                    [("q_proj", d, d), ("k_proj", d, 1024), ("v_proj", d, 1024),
                     ("o_proj", d, d), ("gate_proj", d, 28672), ("up_proj", d, 28672),
                     ("down_proj", 28672, d)], "decode")


BUILDERS = {1: tiny, 2: qproj_decode, 3: qkv_prefill, 4: mixed_mlp, 5: block70b}
NAMES = {1: "tiny", 2: "qproj_decode", 3: "qkv_prefill", 4: "mixed_mlp", 5: "block70b"}


def make(config: int) -> Workload:
    """The full-size workload ``config`` (1..5) with its own seed (config - 1)."""
    return BUILDERS[config]()


def make_small(config: int) -> Workload:
    """A reduced-row variant of ``config`` with the same structure, for oracle parity.

    Row counts are cut so the fp64 oracle finishes in seconds while segments still
    span several tiles and end on ragged tails.
    """
    if config == 1:
        return tiny()
    if config == 2:
        return qproj_decode(n_rows=96)
    if config == 3:
        return qkv_prefill(lo=40, hi=300)
    if config == 4:
        return mixed_mlp(n_decode=64, prefill_len=133, n_prefill=2)
    if config == 5:
        return block70b(n_rows=80)
    raise ValueError(config)


def random_case(seed: int, n_rows: int, d_in: int, d_out: int, n_slots: int,
                ranks, base_frac: float = 0.1, alpha: Optional[float] = None,
                shuffle: bool = True, r_max: Optional[int] = None) -> Workload:
    """A small random workload for edge-case sweeps (ranks drawn from ``ranks``)."""
    rng = np.random.default_rng(seed)
    slot_rank = rng.choice(np.asarray(ranks, np.int32), size=n_slots).astype(np.int32)
    row_slot = rng.integers(0, n_slots, size=n_rows).astype(np.int32)
    if not shuffle:
        row_slot = np.sort(row_slot).astype(np.int32)
    row_slot = _base_mask(rng, row_slot, base_frac)
    alphas = (2.0 * slot_rank if alpha is None else np.full(n_slots, alpha)).astype(np.float64)
    if r_max is None:
        r_max = next(b for b in RANK_BUCKETS if b >= int(slot_rank.max()))
    return Workload(f"random{seed}", seed, n_slots, int(r_max), slot_rank, alphas, row_slot,
                    [("proj", d_in, d_out)], "mixed")
