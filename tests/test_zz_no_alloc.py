"""mlora_apply_noalloc: the fused apply for callers that cannot allocate device memory.

Callers such as a serving engine that has reserved nearly all of HBM up front and
hands out memory only from its own allocator cannot let the library grow a
workspace with cudaMalloc, as mlora_apply does for long segments.  The no-allocation
entry point keeps that workspace in a fixed 4 MiB array inside the library instead.
These tests call it through the C ABI and check that it gives what mlora_apply
gives, and what the fp64 oracle gives, within the parity tolerance, on calls in a
row (each finds the previous call's H values still in the shared array); that its
first call after pool creation takes no device memory (the array is reserved when
the pool is created); that a batch needing more scratch than the array holds is
refused with nothing written; and that a large batch that never uses the scratch
(decode rows only) is not refused.

The file is named so that pytest collects it last; it also passes on its own in a
fresh process, where its first call does the per-device set-up.
"""
import numpy as np
import pytest
import torch

import oracle
import segmented_rank_gemm_02_b200 as mlora
import workloads as wl
from gpu_harness import DEVICE, assert_close, bf16_f64, free
from segmented_rank_gemm_02_b200 import staging

pytestmark = pytest.mark.gpu


def _pair(W, proj):
    """Y after mlora_apply and after mlora_apply_noalloc on the same staged inputs."""
    st = staging.upload(W, proj, DEVICE)
    Y0 = st["Y"].clone()
    mlora.apply(st["pool"], st["segs"], st["X"], st["Y"])
    assert st["pool"].check() == 0
    Y_ref = mlora.bf16_bits(st["Y"])
    Y = Y0.clone()
    mlora.apply_noalloc(st["pool"], st["segs"], st["X"], Y)
    assert st["pool"].check() == 0
    return mlora.bf16_bits(Y), Y_ref, st


def _long_segments(W) -> int:
    lengths = np.bincount(W.row_slot[W.row_slot >= 0])
    return int((lengths >= 128).sum())


def test_first_call_after_pool_creation_takes_no_device_memory():
    # the path's kernels are launched once through mlora_apply first (their first
    # launch may make the driver size their local memory); then the first
    # no-allocation call must leave the device's free memory unchanged
    W = wl.make_small(3)
    proj = W.projection(0)
    st = staging.upload(W, proj, DEVICE)
    Y = st["Y"].clone()
    mlora.apply(st["pool"], st["segs"], st["X"], Y)
    assert st["pool"].check() == 0
    Y.copy_(st["Y"])
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    mlora.apply_noalloc(st["pool"], st["segs"], st["X"], Y)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert st["pool"].check() == 0
    assert free_after == free_before
    assert_close(mlora.bf16_bits(Y), oracle.reference(W, proj), "first no-allocation call")
    del st
    free()


def test_noalloc_matches_apply_and_oracle_calls_in_a_row():
    # consecutive calls with different shapes and inputs; each finds the previous
    # call's values in the shared array
    calls = [(3, 0), (4, 2), (4, 0), (3, 0)]
    for i, (cfg, j) in enumerate(calls):
        W = wl.make_small(cfg)
        assert _long_segments(W) > 0      # the workspace is really used
        proj = W.projection(j)
        Y, Y_ref, st = _pair(W, proj)
        assert_close(Y, bf16_f64(Y_ref), f"call {i + 1}: cfg{cfg}/{proj.name} vs mlora_apply")
        assert_close(Y, oracle.reference(W, proj), f"call {i + 1}: cfg{cfg}/{proj.name} vs oracle")
        base = np.nonzero(W.row_slot < 0)[0]
        assert np.array_equal(Y[base], proj.Y0[base])
        del st, proj
        free()


def test_noalloc_rejects_batch_beyond_scratch():
    # rank-64 pool, rows sorted by slot (two runs of consecutive rows, so the batch
    # takes the long-segment kernels): 16384 grouped rows fit the 4 MiB array, 16400
    # do not
    W = wl.random_case(11, n_rows=16400, d_in=64, d_out=64, n_slots=2, ranks=[64],
                       base_frac=0.0, shuffle=False)
    proj = W.projection(0)
    st = staging.upload(W, proj, DEVICE)
    assert st["meta"]["max_segment_rows"] >= 128
    Y = st["Y"].clone()
    with pytest.raises(mlora.MloraError) as e:
        mlora.apply_noalloc(st["pool"], st["segs"], st["X"], Y)
    assert e.value.status == mlora.ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.equal(Y, st["Y"])
    del st
    free()


def test_noalloc_large_decode_batch_needs_no_scratch():
    # the same size with rows in random order: no run of consecutive rows reaches the
    # long-segment kernels, nothing uses the array, and the call is accepted
    W = wl.random_case(12, n_rows=16400, d_in=64, d_out=64, n_slots=2, ranks=[64],
                       base_frac=0.1, shuffle=True)
    proj = W.projection(0)
    Y, Y_ref, st = _pair(W, proj)
    assert st["meta"]["max_segment_rows"] < 128
    assert_close(Y, bf16_f64(Y_ref), "large decode batch vs mlora_apply")
    rows = np.arange(0, W.n_rows, 97)
    assert_close(Y[rows], oracle.reference(W, proj, rows=rows), "large decode batch vs oracle")
    del st
    free()
