"""fp64 CPU oracle for the heterogeneous-batch LoRA branch.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product package never
imports this module, and this module never imports the product package.

Two parts:

* ``group_rows`` -- the grouping step, written in numpy from the metadata example
  on the page "Multi-LoRA Serving: adapter batching" (charlestar.github.io, section
  "What metadata a segmented kernel needs"): rows are grouped by adapter slot into
  segments; segments appear in the order their slot first appears among the rows
  and keep the rows' original order inside, so the page's batch (rows 0-3 on A,
  4-5 base, 6-10 on B, 11 on C) gives offsets [0, 4, 6, 11, 12], slots
  [A, base, B, C] and the identity row mapping.
* the contraction (``apply_segments``, ``apply_rows``, ``shrink``, ``expand``) --
  thin ctypes wrappers over ``oracle.c`` (plain C, fp64, OpenMP over rows).

Arrays of bf16 values are ``uint16`` bit patterns; Y is handled in fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

BAD_OFFSETS, BAD_SLOT, BAD_RANK, BAD_ROW, SLOT_EMPTY = 1, 2, 4, 8, 16

_u16p = ctypes.POINTER(ctypes.c_uint16)
_i32p = ctypes.POINTER(ctypes.c_int32)
_f64p = ctypes.POINTER(ctypes.c_double)
_u16pp = ctypes.POINTER(_u16p)


def build(force: bool = False, out: str = _LIB_PATH, defines: Sequence[str] = ()) -> str:
    """Compile oracle.c with gcc (-O2, OpenMP) into a shared library."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(_SRC) and not defines):
        return out
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-Wall",
           *[f"-D{d}" for d in defines], "-o", out, _SRC]
    subprocess.run(cmd, check=True)
    return out


def _declare(lib):
    lib.orc_apply_segments.restype = ctypes.c_int
    lib.orc_apply_segments.argtypes = [
        ctypes.c_int, ctypes.c_int, ctypes.c_int, _u16p, ctypes.c_int64, _f64p, ctypes.c_int64,
        ctypes.c_int, _i32p, _i32p, _i32p, _f64p, ctypes.c_int, _i32p,
        ctypes.c_int, _i32p, _f64p, _u16pp, _u16pp, ctypes.c_int]
    lib.orc_apply_rows.restype = ctypes.c_int
    lib.orc_apply_rows.argtypes = [
        ctypes.c_int, ctypes.c_int, ctypes.c_int, _u16p, ctypes.c_int64, _f64p, ctypes.c_int64,
        _i32p, _f64p, ctypes.c_int, _i32p, _f64p, _u16pp, _u16pp, ctypes.c_int]
    lib.orc_apply_rows_xf64.restype = ctypes.c_int
    lib.orc_apply_rows_xf64.argtypes = [
        ctypes.c_int, ctypes.c_int, ctypes.c_int, _f64p, ctypes.c_int64, _f64p, ctypes.c_int64,
        _i32p, _f64p, ctypes.c_int, _i32p, _f64p, _u16pp, _u16pp, ctypes.c_int]
    lib.orc_shrink.restype = ctypes.c_int
    lib.orc_shrink.argtypes = [
        ctypes.c_int, ctypes.c_int, _u16p, ctypes.c_int64,
        ctypes.c_int, _i32p, _i32p, _i32p, ctypes.c_int, _i32p,
        ctypes.c_int, _i32p, _u16pp, _f64p, ctypes.c_int64, ctypes.c_int]
    lib.orc_expand.restype = ctypes.c_int
    lib.orc_expand.argtypes = [
        ctypes.c_int, ctypes.c_int, _f64p, ctypes.c_int64, _f64p, ctypes.c_int64,
        ctypes.c_int, _i32p, _i32p, _i32p, _f64p, ctypes.c_int, _i32p,
        ctypes.c_int, _i32p, _f64p, _u16pp, ctypes.c_int]
    lib.orc_adapter_params_read.restype = ctypes.c_int64
    lib.orc_adapter_params_read.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.orc_max_threads.restype = ctypes.c_int
    lib.orc_max_threads.argtypes = []
    return lib


def load(path: Optional[str] = None):
    """Load (building if needed) the oracle library; ``path`` loads another build."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build()))
    return _lib


# ---------------------------------------------------------------------------
# small conversions
# ---------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns as float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def _p(a: Optional[np.ndarray], ptype):
    if a is None:
        return None
    return a.ctypes.data_as(ptype)


def _i32(a) -> Optional[np.ndarray]:
    return None if a is None else np.ascontiguousarray(a, dtype=np.int32)


def _f64(a) -> Optional[np.ndarray]:
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _ptr_table(mats: Dict[int, np.ndarray], n_slots: int):
    keep = []
    table = (_u16p * max(n_slots, 1))()
    for s, m in mats.items():
        if 0 <= s < n_slots:
            m = np.ascontiguousarray(m, dtype=np.uint16)
            keep.append(m)
            table[s] = m.ctypes.data_as(_u16p)
    return table, keep


# ---------------------------------------------------------------------------
# grouping (a0)
# ---------------------------------------------------------------------------

def group_rows(row_slot: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Group rows by slot: segments in order of each slot's first appearance,
    rows in their original order inside each segment.

    Returns ``(segment_offsets[S+1], adapter_slots[S], token_indices[n])`` where
    ``token_indices[p]`` is the original row of grouped position ``p``.
    """
    row_slot = np.asarray(row_slot, dtype=np.int64)
    n = row_slot.shape[0]
    if n == 0:
        return np.zeros(1, np.int32), np.zeros(0, np.int32), np.zeros(0, np.int32)
    order_seen = []
    seen = set()
    for s in row_slot.tolist():
        if s not in seen:
            seen.add(s)
            order_seen.append(s)
    position = {s: i for i, s in enumerate(order_seen)}
    key = np.array([position[s] for s in row_slot.tolist()], dtype=np.int64)
    token_indices = np.argsort(key, kind="stable").astype(np.int32)
    counts = np.bincount(key, minlength=len(order_seen))
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return offsets, np.array(order_seen, dtype=np.int32), token_indices


# ---------------------------------------------------------------------------
# the contraction
# ---------------------------------------------------------------------------

def apply_segments(X: np.ndarray, Y0: np.ndarray, offsets, slots, ranks, scales,
                   token_indices, slot_rank, slot_alpha, A: Dict[int, np.ndarray],
                   B: Dict[int, np.ndarray], n_tokens: Optional[int] = None,
                   n_threads: int = 0) -> Tuple[np.ndarray, int]:
    """Segmented formulation.  ``Y0`` may be bf16 bits (uint16) or float64.

    Returns ``(Y fp64 [n_rows, d_out], flags)``.
    """
    lib = load()
    X = np.ascontiguousarray(X, dtype=np.uint16)
    Y = bf16_to_f64(Y0) if Y0.dtype == np.uint16 else np.array(Y0, dtype=np.float64, order="C")
    n_rows, d_in = X.shape
    d_out = Y.shape[1]
    offsets, slots, ranks, ti = _i32(offsets), _i32(slots), _i32(ranks), _i32(token_indices)
    scales = _f64(scales)
    slot_rank, slot_alpha = _i32(slot_rank), _f64(slot_alpha)
    n_slots = slot_rank.shape[0]
    if n_tokens is None:
        n_tokens = int(offsets[-1]) if ti is None else int(ti.shape[0])
    ta, ka = _ptr_table(A, n_slots)
    tb, kb = _ptr_table(B, n_slots)
    flags = lib.orc_apply_segments(
        n_rows, d_in, d_out, _p(X, _u16p), d_in, _p(Y, _f64p), d_out,
        int(slots.shape[0]), _p(offsets, _i32p), _p(slots, _i32p), _p(ranks, _i32p),
        _p(scales, _f64p), int(n_tokens), _p(ti, _i32p), n_slots, _p(slot_rank, _i32p),
        _p(slot_alpha, _f64p), ta, tb, int(n_threads))
    del ka, kb
    return Y, int(flags)


def apply_rows(X: np.ndarray, Y0: np.ndarray, row_slot, row_scale, slot_rank, slot_alpha,
               A: Dict[int, np.ndarray], B: Dict[int, np.ndarray],
               n_threads: int = 0) -> Tuple[np.ndarray, int]:
    """Per-row (gather) formulation over rows in original order."""
    lib = load()
    X = np.ascontiguousarray(X, dtype=np.uint16)
    Y = bf16_to_f64(Y0) if Y0.dtype == np.uint16 else np.array(Y0, dtype=np.float64, order="C")
    n_rows, d_in = X.shape
    d_out = Y.shape[1]
    row_slot, row_scale = _i32(row_slot), _f64(row_scale)
    slot_rank, slot_alpha = _i32(slot_rank), _f64(slot_alpha)
    n_slots = slot_rank.shape[0]
    ta, ka = _ptr_table(A, n_slots)
    tb, kb = _ptr_table(B, n_slots)
    flags = lib.orc_apply_rows(
        n_rows, d_in, d_out, _p(X, _u16p), d_in, _p(Y, _f64p), d_out,
        _p(row_slot, _i32p), _p(row_scale, _f64p), n_slots, _p(slot_rank, _i32p),
        _p(slot_alpha, _f64p), ta, tb, int(n_threads))
    del ka, kb
    return Y, int(flags)


def apply_rows_xf64(X: np.ndarray, Y0: np.ndarray, row_slot, row_scale, slot_rank, slot_alpha,
                    A: Dict[int, np.ndarray], B: Dict[int, np.ndarray],
                    n_threads: int = 0) -> Tuple[np.ndarray, int]:
    """Per-row formulation with the activation given as fp64 values (``X`` float64) and
    ``Y0`` as float64 values: the reference at a quantized base model's dtype boundary,
    where X is an FP8 code times its scale and Y0 an fp16 or fp32 base output."""
    lib = load()
    X = np.array(X, dtype=np.float64, order="C")
    Y = np.array(Y0, dtype=np.float64, order="C")
    n_rows, d_in = X.shape
    d_out = Y.shape[1]
    row_slot, row_scale = _i32(row_slot), _f64(row_scale)
    slot_rank, slot_alpha = _i32(slot_rank), _f64(slot_alpha)
    n_slots = slot_rank.shape[0]
    ta, ka = _ptr_table(A, n_slots)
    tb, kb = _ptr_table(B, n_slots)
    flags = lib.orc_apply_rows_xf64(
        n_rows, d_in, d_out, _p(X, _f64p), d_in, _p(Y, _f64p), d_out,
        _p(row_slot, _i32p), _p(row_scale, _f64p), n_slots, _p(slot_rank, _i32p),
        _p(slot_alpha, _f64p), ta, tb, int(n_threads))
    del ka, kb
    return Y, int(flags)


def base_gemm_apply(X: np.ndarray, W: np.ndarray, row_slot, row_scale, slot_rank, slot_alpha,
                    A: Dict[int, np.ndarray], B: Dict[int, np.ndarray],
                    n_threads: int = 0) -> Tuple[np.ndarray, int]:
    """The base projection and the LoRA branch together (page "Multi-LoRA serving",
    ybb.press ai-applications, section 3.3, W0 x + B(A x) in one kernel; page "Multi-LoRA Serving:
    adapter batching", section "LoRA on one Linear layer", Y = X W^T + s (X A^T) B^T):
    Y[t] = X[t] W^T + s_a (X[t] A_a^T) B_a^T for rows of adapter a, X[t] W^T for base
    rows, in fp64.  ``X`` [n_rows, d_in] and ``W`` [d_out, d_in] (the nn.Linear
    layout) are bf16 bits.  The base term is a library fp64 matmul of the exact bf16
    values; it is then the Y0 of the per-row entry.  Returns ``(Y, flags)``."""
    base = bf16_to_f64(X) @ bf16_to_f64(W).T
    return apply_rows(X, base, row_slot, row_scale, slot_rank, slot_alpha, A, B, n_threads)


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Exact values of FP8 e4m3 codes (1 sign bit, 4 exponent bits with bias 7, 3
    mantissa bits; exponent field 0 is subnormal, 2^-6 * m/8; S.1111.111 is NaN and
    there is no infinity), as float64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = np.where((e == 0xF) & ((c & 0x7) == 0x7), np.nan, val)
    return sign * val


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact values of IEEE binary16 bit patterns as float64."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def shrink(X: np.ndarray, offsets, slots, ranks, token_indices, slot_rank,
           A: Dict[int, np.ndarray], r_cols: int, n_tokens: Optional[int] = None,
           H_init: Optional[np.ndarray] = None, n_threads: int = 0) -> Tuple[np.ndarray, int]:
    """H (fp64 [n_tokens, r_cols], grouped order); untouched entries keep ``H_init``
    (default NaN)."""
    lib = load()
    X = np.ascontiguousarray(X, dtype=np.uint16)
    n_rows, d_in = X.shape
    offsets, slots, ranks, ti = _i32(offsets), _i32(slots), _i32(ranks), _i32(token_indices)
    slot_rank = _i32(slot_rank)
    n_slots = slot_rank.shape[0]
    if n_tokens is None:
        n_tokens = int(offsets[-1]) if ti is None else int(ti.shape[0])
    H = (np.full((n_tokens, r_cols), np.nan) if H_init is None
         else np.array(H_init, dtype=np.float64, order="C"))
    ta, ka = _ptr_table(A, n_slots)
    flags = lib.orc_shrink(
        n_rows, d_in, _p(X, _u16p), d_in, int(slots.shape[0]), _p(offsets, _i32p),
        _p(slots, _i32p), _p(ranks, _i32p), int(n_tokens), _p(ti, _i32p), n_slots,
        _p(slot_rank, _i32p), ta, _p(H, _f64p), r_cols, int(n_threads))
    del ka
    return H, int(flags)


def expand(H: np.ndarray, Y0: np.ndarray, offsets, slots, ranks, scales, token_indices,
           slot_rank, slot_alpha, B: Dict[int, np.ndarray], n_tokens: Optional[int] = None,
           n_threads: int = 0) -> Tuple[np.ndarray, int]:
    """Y0 + s * H B^T scattered to the original rows (fp64)."""
    lib = load()
    H = np.array(H, dtype=np.float64, order="C")
    Y = bf16_to_f64(Y0) if Y0.dtype == np.uint16 else np.array(Y0, dtype=np.float64, order="C")
    n_rows, d_out = Y.shape
    offsets, slots, ranks, ti = _i32(offsets), _i32(slots), _i32(ranks), _i32(token_indices)
    scales = _f64(scales)
    slot_rank, slot_alpha = _i32(slot_rank), _f64(slot_alpha)
    n_slots = slot_rank.shape[0]
    if n_tokens is None:
        n_tokens = int(offsets[-1]) if ti is None else int(ti.shape[0])
    tb, kb = _ptr_table(B, n_slots)
    flags = lib.orc_expand(
        n_rows, d_out, _p(H, _f64p), H.shape[1], _p(Y, _f64p), d_out, int(slots.shape[0]),
        _p(offsets, _i32p), _p(slots, _i32p), _p(ranks, _i32p), _p(scales, _f64p),
        int(n_tokens), _p(ti, _i32p), n_slots, _p(slot_rank, _i32p), _p(slot_alpha, _f64p),
        tb, int(n_threads))
    del kb
    return Y, int(flags)


def adapter_params_read(d_in: int, d_out: int, r: int) -> int:
    return int(load().orc_adapter_params_read(d_in, d_out, r))


def max_threads() -> int:
    return int(load().orc_max_threads())


# ---------------------------------------------------------------------------
# convenience over a workload projection
# ---------------------------------------------------------------------------

def segments_for(workload) -> dict:
    """Grouped metadata for a workload: offsets, slots, ranks, token_indices."""
    offsets, slots, ti = group_rows(workload.row_slot)
    ranks = np.array([0 if s < 0 else int(workload.slot_rank[s]) for s in slots.tolist()],
                     dtype=np.int32)
    return {"offsets": offsets, "slots": slots, "ranks": ranks, "token_indices": ti}


def reference(workload, proj, meta: Optional[dict] = None, rows: Optional[np.ndarray] = None,
              n_threads: int = 0) -> np.ndarray:
    """fp64 reference Y for one projection of a workload.

    ``rows`` restricts the computation to those original rows (for sampled checks
    of full-size workloads); the result then has ``len(rows)`` rows.
    """
    if rows is None:
        meta = meta or segments_for(workload)
        Y, flags = apply_segments(proj.X, proj.Y0, meta["offsets"], meta["slots"], meta["ranks"],
                                  None, meta["token_indices"], workload.slot_rank,
                                  workload.slot_alpha, proj.A, proj.B, n_threads=n_threads)
        assert flags == 0, flags
        return Y
    rows = np.asarray(rows, dtype=np.int64)
    Y, flags = apply_rows(proj.X[rows], proj.Y0[rows], workload.row_slot[rows], None,
                          workload.slot_rank, workload.slot_alpha, proj.A, proj.B,
                          n_threads=n_threads)
    assert flags == 0, flags
    return Y
