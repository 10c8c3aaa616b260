"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare with the fp64 oracle.

Tolerance (the method's stated bar): |gpu - oracle| <= 1e-2 * (1 + |oracle|)
elementwise on bf16 outputs, with the oracle in fp64.  Rows that get no delta
(base-only, uncovered, rejected) must be bit-identical to Y0.  The mapping check
asks more: each adapter row must be four times closer to its own adapter's
result than to the result under any other loaded adapter.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import segmented_rank_gemm_02_b200 as mlora
from segmented_rank_gemm_02_b200 import staging

RTOL = 1e-2

DEVICE = "cuda:0"


def bf16_f64(bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_to_f64(bits)


def assert_close(Y_bits: np.ndarray, ref: np.ndarray, what: str = "") -> None:
    got = bf16_f64(Y_bits)
    err = np.abs(got - ref)
    bound = RTOL * (1.0 + np.abs(ref))
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance, first "
                             f"{[(tuple(i), got[tuple(i)], ref[tuple(i)]) for i in idx]}")


def assert_untouched(Y_bits: np.ndarray, Y0_bits: np.ndarray, rows, what: str = "") -> None:
    rows = np.asarray(rows, dtype=np.int64)
    if rows.size == 0:
        return
    same = np.array_equal(Y_bits[rows], Y0_bits[rows])
    assert same, f"{what}: rows without a delta changed"


def mapping_check(W, proj, rows: np.ndarray, Y_bits_rows: np.ndarray, ref_rows: np.ndarray,
                  candidate_slots=None) -> None:
    """Each row's error must be < 1/4 of its distance to the nearest wrong adapter."""
    rows = np.asarray(rows, dtype=np.int64)
    if rows.size == 0:
        return
    slots = sorted(proj.A) if candidate_slots is None else candidate_slots
    own = W.row_slot[rows]
    err = np.linalg.norm(bf16_f64(Y_bits_rows) - ref_rows, axis=1)
    nearest = np.full(rows.size, np.inf)
    for s in slots:
        alt_slot = np.full(rows.size, s, np.int32)
        Yalt, flags = oracle.apply_rows(proj.X[rows], proj.Y0[rows], alt_slot, None, W.slot_rank,
                                        W.slot_alpha, proj.A, proj.B)
        assert flags == 0
        d = np.linalg.norm(Yalt - ref_rows, axis=1)
        d[own == s] = np.inf
        nearest = np.minimum(nearest, d)
    ok = err < nearest / 4
    assert ok.all(), f"mapping check failed on rows {rows[~ok][:5]}: err {err[~ok][:5]}, " \
                     f"nearest wrong {nearest[~ok][:5]}"


def run_apply(W, proj, meta=None, with_ranks=True, scales=None):
    st = staging.upload(W, proj, DEVICE, meta=meta, with_ranks=with_ranks, scales=scales)
    mlora.apply(st["pool"], st["segs"], st["X"], st["Y"])
    flags = st["pool"].check()
    Y = mlora.bf16_bits(st["Y"])
    return Y, flags, st


def sample_rows(W, n_sample: int, seed: int = 0) -> np.ndarray:
    """Rows to check at full size: the first and last row of every segment and of
    the batch, plus random rows."""
    off, slots, ti = oracle.group_rows(W.row_slot)
    pick = set([0, W.n_rows - 1])
    for g in range(len(slots)):
        pick.add(int(ti[off[g]]))
        pick.add(int(ti[off[g + 1] - 1]))
    rng = np.random.default_rng(seed)
    pick.update(rng.choice(W.n_rows, size=min(n_sample, W.n_rows), replace=False).tolist())
    return np.array(sorted(pick), dtype=np.int64)


def free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
