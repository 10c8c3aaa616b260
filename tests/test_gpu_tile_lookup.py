"""Decode-shaped batches of several waves of tiles, where each cluster runs more than
one tile: a cluster finds its later tiles in a per-segment table its first metadata
scan left in shared memory (at most 256 segments), else by scanning the metadata
again.  Both paths against the oracle on every row, for 8- and 16-row tiles.

Page "Multi-LoRA Serving: adapter batching", section "What metadata a segmented
kernel needs": each tile's segment, first position and slot come from the segment
offsets and slots alone, whichever way the kernel looks them up.
"""
import numpy as np
import pytest

import oracle
import workloads as wl
from gpu_harness import assert_close, assert_untouched, free, run_apply

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_slots,n_rows,ranks", [
    (200, 2400, (8, 16)),      # ~200 segments of ~12 rows: the table, 16-row tiles
    (200, 2400, (16, 32)),     # the table, 8-row tiles (rank-32 pool)
    (600, 3000, (8, 16)),      # ~600 segments: more than the table holds, scans again
])
def test_several_tiles_per_cluster(n_slots, n_rows, ranks):
    # 4096 -> 2048: clusters of six CTAs; scattered decode rows, far more tiles than the
    # clusters that fit at once (the 128-thread kernel)
    W = wl.random_case(70 + n_slots + ranks[-1], n_rows, 4096, 2048, n_slots, ranks, base_frac=0.05)
    proj = W.projection(0)
    Y, flags, st = run_apply(W, proj)
    assert flags == 0
    n_seg = int(np.count_nonzero(st["meta"]["slots"] >= 0))
    assert (n_seg > 256) == (n_slots > 256)
    ref = oracle.reference(W, proj)
    assert_close(Y, ref, f"{n_slots} slots, ranks {ranks}")
    assert_untouched(Y, proj.Y0, np.nonzero(W.row_slot < 0)[0], "base rows")
    del st
    free()
