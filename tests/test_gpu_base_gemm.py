"""The base projection and the LoRA delta in one pass (mlora_base_gemm_apply), against
the oracle.

Page "Multi-LoRA serving" (ybb.press ai-applications), section 3.3 (W0 x + B(A x)
fused into one kernel): Y = X W^T + s (X A^T) B^T for adapter rows and X W^T for every other row,
accumulated in fp32 and rounded to bf16 once.  The oracle is the fp64 per-row entry
with Y0 = X W^T computed in fp64 from the exact bf16 values (oracle.base_gemm_apply).
Every element must satisfy |gpu - oracle| <= 1e-2 (1 + |oracle|), base rows included;
Y starts as NaN so that a row the kernel fails to write shows.
"""
import numpy as np
import pytest
import torch

import oracle
import segmented_rank_gemm_02_b200 as mlora
import workloads as wl
from gpu_harness import DEVICE, RTOL, free
from segmented_rank_gemm_02_b200 import DeviceSegments, build_segments, staging

pytestmark = pytest.mark.gpu


def _nan_output(n_rows, d_out):
    return torch.full((n_rows, d_out), float("nan"), dtype=torch.bfloat16, device=DEVICE)


def _check(got_bits, ref, what):
    got = oracle.bf16_to_f64(got_bits)
    assert not np.isnan(got).any(), f"{what}: rows left unwritten"
    err = np.abs(got - ref)
    bad = err > RTOL * (1 + np.abs(ref))
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements out of tolerance, worst "
                           f"{float((err / (1 + np.abs(ref))).max())}")


def _run(W, proj, Wb, meta=None):
    st = staging.upload(W, proj, DEVICE, meta=meta)
    Wd = mlora.as_bf16_tensor(Wb, DEVICE)
    Y = _nan_output(W.n_rows, proj.d_out)
    mlora.base_gemm_apply(st["pool"], st["segs"], st["X"], Wd, Y)
    assert st["pool"].check() == 0
    return st, Y


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_base_gemm_workloads(cfg):
    W = wl.make_small(cfg)
    proj = W.projection(0)
    Wb = W.base_weight(0)
    st, Y = _run(W, proj, Wb)
    ref, flags = oracle.base_gemm_apply(proj.X, Wb, W.row_slot, None, W.slot_rank, W.slot_alpha, proj.A, proj.B)
    assert flags == 0
    _check(mlora.bf16_bits(Y), ref, W.name)
    del st
    free()


@pytest.mark.parametrize("shuffle", [True, False])
def test_base_gemm_ragged_shapes_and_all_buckets(shuffle):
    # rows, d_in and d_out off the tile sizes (300 rows, d_in 200, d_out 200 < 256),
    # every rank bucket with odd ranks; rows scattered (many slots per 128-row block)
    # or sorted (runs)
    W = wl.random_case(23, 300, 200, 200, 7, (1, 7, 12, 24, 40, 64), shuffle=shuffle)
    proj = W.projection(0)
    Wb = W.base_weight(0)
    st, Y = _run(W, proj, Wb)
    ref, _ = oracle.base_gemm_apply(proj.X, Wb, W.row_slot, None, W.slot_rank, W.slot_alpha, proj.A, proj.B)
    _check(mlora.bf16_bits(Y), ref, "ragged")
    del st
    free()


@pytest.mark.parametrize("n_rows,d_out", [(9472, 512), (2048, 8448), (4096, 6000), (600, 4096)])
def test_base_gemm_tile_widths(n_rows, d_out):
    # shapes for which the host picks each tile width on a full B200 (256 columns for
    # the first and last, 512 for the others: one with a last tile whose second half
    # lies wholly past d_out, one with a ragged second half); rows sorted into runs,
    # several slots per 256-row block
    W = wl.random_case(26, n_rows, 256, d_out, 5, (16, 64), shuffle=False)
    proj = W.projection(0)
    Wb = W.base_weight(0)
    st, Y = _run(W, proj, Wb)
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([np.arange(0, n_rows, 97), rng.choice(n_rows, 64, replace=False),
                                     [n_rows - 1]]))
    ref, _ = oracle.base_gemm_apply(proj.X[rows], Wb, W.row_slot[rows], None, W.slot_rank, W.slot_alpha,
                                    proj.A, proj.B)
    _check(mlora.bf16_bits(Y)[rows], ref, f"{n_rows}x{d_out}")
    del st
    free()


def test_base_gemm_without_segments_is_the_base_projection():
    W = wl.random_case(24, 130, 64, 264, 3, (16,))
    proj = W.projection(0)
    Wb = W.base_weight(0)
    meta = {"offsets": np.zeros(1, np.int32), "slots": np.zeros(0, np.int32), "ranks": np.zeros(0, np.int32),
            "token_indices": np.zeros(0, np.int32), "n_tokens": 0}
    st, Y = _run(W, proj, Wb, meta=meta)
    base = oracle.bf16_to_f64(proj.X) @ oracle.bf16_to_f64(Wb).T
    _check(mlora.bf16_bits(Y), base, "no segments")
    del st
    free()


def test_base_gemm_rejected_and_uncovered_rows_get_the_base_projection():
    W = wl.random_case(25, 200, 96, 136, 4, (8, 16))
    proj = W.projection(0)
    Wb = W.base_weight(0)
    pool = staging.make_pool(proj.d_in, proj.d_out, W.n_slots, W.r_max, W.slot_rank, W.slot_alpha, proj.A, proj.B)
    meta = build_segments(W.row_slot, pool)
    # drop the last segment (its rows are then covered by nothing) and point another
    # at a slot that holds no adapter
    n_seg = len(meta["slots"])
    keep = n_seg - 1
    last_rows = meta["token_indices"][meta["offsets"][keep]:meta["offsets"][n_seg]]
    meta2 = {"offsets": meta["offsets"][:keep + 1].copy(), "slots": meta["slots"][:keep].copy(),
             "ranks": meta["ranks"][:keep].copy(), "token_indices": meta["token_indices"][:meta["offsets"][keep]].copy()}
    meta2["n_tokens"] = int(meta2["offsets"][-1])
    g_bad = next(g for g in range(keep) if meta2["slots"][g] >= 0)
    bad_rows = meta2["token_indices"][meta2["offsets"][g_bad]:meta2["offsets"][g_bad + 1]]
    pool.clear_slot(int(meta2["slots"][g_bad]))
    segs = DeviceSegments(meta2, W.n_rows, DEVICE)
    X = mlora.as_bf16_tensor(proj.X, DEVICE)
    Wd = mlora.as_bf16_tensor(Wb, DEVICE)
    Y = _nan_output(W.n_rows, proj.d_out)
    mlora.base_gemm_apply(pool, segs, X, Wd, Y)
    assert pool.check() & mlora.FLAG_SLOT_EMPTY
    row_slot = W.row_slot.copy()
    row_slot[last_rows] = -1
    row_slot[bad_rows] = -1
    ref, _ = oracle.base_gemm_apply(proj.X, Wb, row_slot, None, W.slot_rank, W.slot_alpha, proj.A, proj.B)
    _check(mlora.bf16_bits(Y), ref, "rejected / uncovered")
    free()


def test_base_gemm_full_size_prefill_sampled_rows():
    # the full qkv_prefill workload (8 requests of 128..2048 rows, rank 64, d 4096 ->
    # 6144), as the benchmark runs it; sampled rows checked against the oracle
    W = wl.make(3)
    proj = W.projection(0)
    Wb = W.base_weight(0)
    st, Y = _run(W, proj, Wb)
    meta = st["meta"]
    starts = meta["token_indices"][meta["offsets"][:-1]]
    ends = meta["token_indices"][meta["offsets"][1:] - 1]
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([starts, ends, [0, 127, 128, W.n_rows - 1],
                                     rng.choice(W.n_rows, 40, replace=False)]))
    ref, _ = oracle.base_gemm_apply(proj.X[rows], Wb, W.row_slot[rows], None, W.slot_rank, W.slot_alpha,
                                    proj.A, proj.B)
    _check(mlora.bf16_bits(Y)[rows], ref, "qkv_prefill sampled")
    del st
    free()


def test_base_gemm_argument_errors():
    W = wl.make_small(1)
    proj = W.projection(0)
    st = staging.upload(W, proj, DEVICE)
    Wd = mlora.as_bf16_tensor(W.base_weight(0), DEVICE)
    Y = _nan_output(W.n_rows, proj.d_out)
    wide = torch.zeros((proj.d_out, proj.d_in + 4), dtype=torch.bfloat16, device=DEVICE)[:, :proj.d_in]
    with pytest.raises(mlora.MloraError) as e:
        mlora.base_gemm_apply(st["pool"], st["segs"], st["X"], wide, Y)   # ldw not a multiple of 8
    assert e.value.status == mlora.ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.isnan(Y.float()).all()
    del st
    free()
