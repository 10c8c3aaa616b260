"""16-row decode tiles (batches of long decode segments at rank <= 16) against the oracle.

The decode-shaped kernel takes 16 grouped positions per tile (both halves of the m16
MMA tile) when a batch averages at least 8 rows per segment and the pool's largest
rank bucket is 16 or less; otherwise 8.  These cases force the 16-row path with
scattered rows (so no segment goes to the long-segment kernels) and check every
element against the oracle (|gpu - oracle| <= 1e-2 (1 + |oracle|)), rows without a
delta bit-identical, for single and fused projections, odd ranks and ragged tails.
"""
import numpy as np
import pytest

import oracle
import segmented_rank_gemm_02_b200 as mlora
import workloads as wl
from gpu_harness import DEVICE, assert_close, assert_untouched, free, run_apply
from segmented_rank_gemm_02_b200 import staging

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seed,n_rows,n_slots,ranks", [
    (41, 600, 20, (1, 8, 12, 16)),      # ~30 rows per segment, every tail length
    (42, 350, 37, (16,)),               # ~9-10 rows per segment: tiles of 9..16 rows
    (43, 900, 8, (3, 8)),               # rank bucket 8 only
])
def test_tall_tiles_single_projection(seed, n_rows, n_slots, ranks):
    W = wl.random_case(seed, n_rows, 512, 384, n_slots, ranks, base_frac=0.1, shuffle=True)
    meta = mlora.build_segments(W.row_slot)
    assert W.n_rows >= 8 * len(meta["slots"])   # the batch takes 16-row tiles
    proj = W.projection(0)
    Y, flags, st = run_apply(W, proj)
    assert flags == 0
    ref = oracle.reference(W, proj)
    assert_close(Y, ref, f"tall tiles seed {seed}")
    assert_untouched(Y, proj.Y0, np.nonzero(W.row_slot < 0)[0], "base rows")
    del st
    free()


def test_tall_tiles_fused_projections():
    W = wl.random_case(44, 512, 512, 256, 16, (8, 16), base_frac=0.05, shuffle=True)
    W.proj_shapes = [("q_proj", 512, 256), ("k_proj", 512, 128)]
    q, k = W.projection(0), W.projection(1)
    k.X = q.X
    pools = [staging.make_pool(512, pr.d_out, W.n_slots, W.r_max, W.slot_rank, W.slot_alpha, pr.A, pr.B)
             for pr in (q, k)]
    segs = mlora.DeviceSegments(mlora.build_segments(W.row_slot, pools[0]), W.n_rows, DEVICE)
    X = mlora.as_bf16_tensor(q.X, DEVICE)
    Ys = [mlora.as_bf16_tensor(pr.Y0, DEVICE) for pr in (q, k)]
    mlora.apply_multi(pools, segs, X, Ys)
    base = np.nonzero(W.row_slot < 0)[0]
    for pool, pr, Y in zip(pools, (q, k), Ys):
        assert pool.check() == 0
        got = mlora.bf16_bits(Y)
        assert_close(got, oracle.reference(W, pr), f"fused {pr.name}")
        assert_untouched(got, pr.Y0, base, f"fused {pr.name}")
    free()


def test_tall_tiles_bad_rows_are_skipped():
    # one token index out of range inside a long segment: that row is skipped and
    # flagged, every other row of the tile still gets its delta
    W = wl.random_case(45, 400, 256, 256, 6, (16,), base_frac=0.0, shuffle=True)
    proj = W.projection(0)
    pool = staging.make_pool(256, 256, W.n_slots, W.r_max, W.slot_rank, W.slot_alpha, proj.A, proj.B)
    meta = mlora.build_segments(W.row_slot, pool)
    bad_pos = int(meta["offsets"][0]) + 9            # position 9 of the first tile: a row g + 8
    dropped = int(meta["token_indices"][bad_pos])
    meta["token_indices"] = meta["token_indices"].copy()
    meta["token_indices"][bad_pos] = W.n_rows + 5
    segs = mlora.DeviceSegments(meta, W.n_rows, DEVICE)
    X = mlora.as_bf16_tensor(proj.X, DEVICE)
    Y = mlora.as_bf16_tensor(proj.Y0, DEVICE)
    mlora.apply(pool, segs, X, Y)
    assert pool.check() & mlora.FLAG_BAD_ROW
    row_slot = W.row_slot.copy()
    row_slot[dropped] = -1
    ref, _ = oracle.apply_rows(proj.X, proj.Y0, row_slot, None, W.slot_rank, W.slot_alpha, proj.A, proj.B)
    got = mlora.bf16_bits(Y)
    assert_close(got, ref, "bad row skipped")
    assert_untouched(got, proj.Y0, [dropped], "dropped row")
    free()
