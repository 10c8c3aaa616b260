"""Move host-side adapters and activations into the library's device structures.

Convenience for callers that hold adapters as PEFT-layout bf16 arrays (uint16 bit
patterns): fill a pool, build the segment metadata with the library's host
grouping helper, and copy X / Y0 to the device.  No LoRA arithmetic happens here.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from . import DeviceSegments, Pool, as_bf16_tensor, build_segments


def make_pool(d_in: int, d_out: int, n_slots: int, r_max: int, slot_rank: np.ndarray,
              slot_alpha: np.ndarray, A: Dict[int, np.ndarray], B: Dict[int, np.ndarray],
              stream=None) -> Pool:
    """A pool with every slot present in ``A``/``B`` loaded at its rank and alpha."""
    pool = Pool(d_in, d_out, n_slots, r_max)
    for s in sorted(A):
        pool.load_slot(int(s), int(slot_rank[s]), float(slot_alpha[s]), A[s], B[s], stream=stream)
    return pool


def upload(workload, proj, device, pool: Optional[Pool] = None, meta: Optional[dict] = None,
           with_ranks: bool = True, scales=None) -> dict:
    """Pool, device metadata, X and Y (= Y0) tensors for one projection of a workload."""
    if pool is None:
        pool = make_pool(proj.d_in, proj.d_out, workload.n_slots, workload.r_max,
                         workload.slot_rank, workload.slot_alpha, proj.A, proj.B)
    if meta is None:
        meta = build_segments(workload.row_slot, pool)
        if not with_ranks:
            meta.pop("ranks", None)
    segs = DeviceSegments(meta, workload.n_rows, device, scales=scales)
    X = as_bf16_tensor(proj.X, device)
    Y = as_bf16_tensor(proj.Y0, device)
    return {"pool": pool, "segs": segs, "meta": meta, "X": X, "Y": Y}
