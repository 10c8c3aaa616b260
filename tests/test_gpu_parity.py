"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
five workloads -- every element of reduced-row versions, and sampled rows plus
every untouched row of the full-size versions."""
import numpy as np
import pytest

import oracle
import workloads as wl
from gpu_harness import (assert_close, assert_untouched, free, mapping_check, run_apply,
                         sample_rows)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_apply_reduced_workload(cfg):
    W = wl.make_small(cfg)
    base = np.nonzero(W.row_slot < 0)[0]
    adapter_rows = np.nonzero(W.row_slot >= 0)[0]
    for j in range(len(W.proj_shapes)):
        proj = W.projection(j)
        Y, flags, st = run_apply(W, proj)
        assert flags == 0
        ref = oracle.reference(W, proj)
        assert_close(Y, ref, f"cfg{cfg}/{proj.name}")
        assert_untouched(Y, proj.Y0, base, f"cfg{cfg}/{proj.name}")
        pick = adapter_rows[:: max(1, adapter_rows.size // 24)]
        mapping_check(W, proj, pick, Y[pick], ref[pick])
        del st
        free()


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_apply_full_workload_sampled(cfg):
    W = wl.make(cfg)
    base = np.nonzero(W.row_slot < 0)[0]
    rows = sample_rows(W, 24, seed=cfg)
    for j in range(len(W.proj_shapes)):
        proj = W.projection(j)
        Y, flags, st = run_apply(W, proj)
        assert flags == 0
        ref = oracle.reference(W, proj, rows=rows)
        assert_close(Y[rows], ref, f"cfg{cfg}/{proj.name}")
        assert_untouched(Y, proj.Y0, base, f"cfg{cfg}/{proj.name}")
        del st, proj
        free()


def test_apply_is_deterministic():
    W = wl.make_small(2)
    proj = W.projection(0)
    Y1, f1, _ = run_apply(W, proj)
    Y2, f2, _ = run_apply(W, proj)
    assert f1 == f2 == 0
    assert np.array_equal(Y1, Y2)
