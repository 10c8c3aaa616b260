"""mlora_apply_multi: one launch applying the deltas of several projections that read
the same input rows (q/k/v, gate/up; page "Multi-LoRA Serving: adapter batching",
section "An adapter is not one contiguous weight": an adapter carries its own A and
B for every target module of a layer).

Each projection k has its own pool (same d_in and slot numbering) and output Y_k;
the expected result is the oracle applied to every projection with the shared X.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import segmented_rank_gemm_02_b200 as mlora
import workloads as wl
from gpu_harness import DEVICE, assert_close, assert_untouched, free, mapping_check, sample_rows
from segmented_rank_gemm_02_b200 import staging

pytestmark = pytest.mark.gpu


def fused_case(seed, n_rows, d_in, d_outs, n_slots, ranks, base_frac=0.1, shuffle=True):
    """A random batch and one projection per d_out, all reading projection 0's X."""
    W = wl.random_case(seed, n_rows, d_in, d_outs[0], n_slots, ranks, base_frac=base_frac,
                       shuffle=shuffle)
    W = dataclasses.replace(W, proj_shapes=[(f"p{k}", d_in, d) for k, d in enumerate(d_outs)],
                            _proj_cache={})
    projs = [W.projection(k) for k in range(len(d_outs))]
    return W, [dataclasses.replace(p, X=projs[0].X) for p in projs]


def make_pools(W, projs, r_max=None):
    return [staging.make_pool(p.d_in, p.d_out, W.n_slots, r_max or W.r_max, W.slot_rank,
                              W.slot_alpha, p.A, p.B) for p in projs]


def run_fused(W, projs, pools=None, meta=None):
    pools = pools or make_pools(W, projs)
    meta = meta if meta is not None else mlora.build_segments(W.row_slot, pools[0])
    segs = mlora.DeviceSegments(meta, W.n_rows, DEVICE)
    X = mlora.as_bf16_tensor(projs[0].X, DEVICE)
    Ys = [mlora.as_bf16_tensor(p.Y0, DEVICE) for p in projs]
    mlora.apply_multi(pools, segs, X, Ys)
    flags = [pl.check() for pl in pools]
    return [mlora.bf16_bits(Y) for Y in Ys], flags, pools


def check_all(W, projs, Ys, what):
    base = np.nonzero(W.row_slot < 0)[0]
    for k, (p, Y) in enumerate(zip(projs, Ys)):
        ref = oracle.reference(W, p)
        assert_close(Y, ref, f"{what}: projection {k}")
        assert_untouched(Y, p.Y0, base, f"{what}: projection {k}")


@pytest.mark.parametrize("d_outs,ranks,shuffle", [
    ((1024, 256, 256), (8, 16, 32), True),     # q/k/v-like, mixed ranks, scattered rows
    ((512, 512), (16,), True),                 # gate/up-like
    ((384, 128, 256, 640), (8, 64), True),     # the maximum of four projections
    ((256,), (16, 32), True),                  # one projection through the fused kernel
])
def test_fused_decode_matches_oracle(d_outs, ranks, shuffle):
    W, projs = fused_case(41, 230, 1024, d_outs, 6, ranks, shuffle=shuffle)
    Ys, flags, _ = run_fused(W, projs)
    assert flags == [0] * len(projs)
    check_all(W, projs, Ys, f"d_outs {d_outs}")
    rows = np.nonzero(W.row_slot >= 0)[0][:12]
    for p, Y in zip(projs, Ys):
        mapping_check(W, p, rows, Y[rows], oracle.reference(W, p, rows=rows))
    free()


def test_fused_with_long_segments():
    # sorted rows without base rows: segments of >= 128 consecutive rows go to the
    # long-segment kernels, once per projection; the short ones to the fused launch
    W, projs = fused_case(42, 700, 512, (768, 256), 5, (16, 64), base_frac=0.0, shuffle=False)
    meta = mlora.build_segments(W.row_slot)
    assert meta["max_segment_rows"] >= 128
    Ys, flags, _ = run_fused(W, projs)
    assert flags == [0, 0]
    check_all(W, projs, Ys, "long + short")
    free()


@pytest.mark.parametrize("d_outs,ranks", [
    ((512, 384, 256), (8, 16, 32)),            # three projections in one long shrink
    ((256, 512, 128, 384), (16, 64)),          # four: the largest fused shrink
])
def test_fused_long_shrink_several_projections(d_outs, ranks):
    # segments of >= 128 consecutive rows: one shrink launch computes H for every
    # projection (X's rows read once), then each projection's expand
    W, projs = fused_case(46, 900, 512, d_outs, 4, ranks, base_frac=0.0, shuffle=False)
    assert mlora.build_segments(W.row_slot)["max_segment_rows"] >= 128
    Ys, flags, _ = run_fused(W, projs)
    assert flags == [0] * len(projs)
    check_all(W, projs, Ys, f"long, {len(d_outs)} projections")
    free()


def test_fused_long_segments_pools_with_different_rmax():
    # rank buckets differ between the pools: each projection takes its own shrink
    W, projs = fused_case(47, 700, 512, (512, 384), 4, (8, 16), base_frac=0.0, shuffle=False)
    pools = [make_pools(W, projs[:1], r_max=16)[0], make_pools(W, projs[1:], r_max=64)[0]]
    Ys, flags, _ = run_fused(W, projs, pools=pools)
    assert flags == [0, 0]
    check_all(W, projs, Ys, "long, r_max 16 / 64")
    free()


def test_fused_long_segments_slot_ranks_differ_between_pools():
    # an adapter may use another rank in each target module; with equal pool buckets one
    # shrink launch serves both projections, and each H must come from its own rank
    W, projs = fused_case(48, 900, 512, (512, 384), 4, (16, 32, 64), base_frac=0.0, shuffle=False)
    ranks1 = np.array([r // 2 + 3 if r > 0 else r for r in W.slot_rank], dtype=W.slot_rank.dtype)
    A1 = {s: np.ascontiguousarray(a[:ranks1[s]]) for s, a in projs[1].A.items()}
    B1 = {s: np.ascontiguousarray(b[:, :ranks1[s]]) for s, b in projs[1].B.items()}
    W1 = dataclasses.replace(W, slot_rank=ranks1, _proj_cache={})
    p1 = dataclasses.replace(projs[1], A=A1, B=B1)
    pools = [staging.make_pool(512, 512, W.n_slots, 64, W.slot_rank, W.slot_alpha, projs[0].A, projs[0].B),
             staging.make_pool(512, 384, W.n_slots, 64, ranks1, W.slot_alpha, A1, B1)]
    meta = mlora.build_segments(W.row_slot)
    meta.pop("ranks", None)   # the metadata cannot carry two ranks per segment
    assert meta["max_segment_rows"] >= 128
    Ys, flags, _ = run_fused(W, [projs[0], p1], pools=pools, meta=meta)
    assert flags == [0, 0]
    assert_close(Ys[0], oracle.reference(W, projs[0]), "projection 0, its own ranks")
    assert_close(Ys[1], oracle.reference(W1, p1), "projection 1, other ranks")
    free()


def test_fused_pools_with_different_rmax():
    # projection 1's pool is built for rank 64, projection 0's for rank 16
    W, projs = fused_case(43, 150, 512, (512, 384), 4, (8, 16))
    pools = [make_pools(W, projs[:1], r_max=16)[0], make_pools(W, projs[1:], r_max=64)[0]]
    Ys, flags, _ = run_fused(W, projs, pools=pools)
    assert flags == [0, 0]
    check_all(W, projs, Ys, "r_max 16 / 64")
    free()


def test_fused_stale_slot_reported_by_its_pool():
    W, projs = fused_case(44, 120, 512, (512, 256), 3, (16,))
    pools = make_pools(W, projs)
    meta = mlora.build_segments(W.row_slot, pools[0])
    meta["generations"] = np.array([0 if s < 0 else pools[0].generation(int(s)) for s in meta["slots"]],
                                   np.uint32)
    # slot 1 of projection 1's pool is reloaded after the batch was built
    rng = np.random.default_rng(9)
    A2 = wl.f32_to_bf16_bits(rng.standard_normal((16, 512), dtype=np.float32) * 0.02)
    B2 = wl.f32_to_bf16_bits(rng.standard_normal((256, 16), dtype=np.float32) * 0.02)
    pools[1].load_slot(1, 16, float(W.slot_alpha[1]), A2, B2)
    Ys, flags, _ = run_fused(W, projs, pools=pools, meta=meta)
    assert flags[0] == 0
    assert flags[1] & mlora.FLAG_STALE_SLOT
    check_all(W, projs[:1], Ys[:1], "fresh pool")
    stale = np.nonzero(W.row_slot == 1)[0]
    assert stale.size > 0
    assert_untouched(Ys[1], projs[1].Y0, stale, "stale slot")
    keep = np.nonzero(W.row_slot != 1)[0]
    assert_close(Ys[1][keep], oracle.reference(W, projs[1])[keep], "other slots")
    free()


def test_fused_bad_metadata_goes_to_first_pool():
    W, projs = fused_case(45, 64, 256, (256, 128), 3, (8,))
    pools = make_pools(W, projs)
    meta = mlora.build_segments(W.row_slot, pools[0])
    g = int(np.nonzero(meta["slots"] >= 0)[0][0])
    meta["slots"] = meta["slots"].copy()
    meta["slots"][g] = 99   # out of range: skipped, flagged while scanning
    Ys, flags, _ = run_fused(W, projs, pools=pools, meta=meta)
    assert flags[0] & mlora.FLAG_BAD_SLOT
    bad_rows = meta["token_indices"][meta["offsets"][g]:meta["offsets"][g + 1]]
    for p, Y in zip(projs, Ys):
        assert_untouched(Y, p.Y0, bad_rows, "rejected segment")
    free()


def test_fused_argument_errors():
    W, projs = fused_case(46, 32, 256, (256, 256), 2, (8,))
    pools = make_pools(W, projs)
    meta = mlora.build_segments(W.row_slot, pools[0])
    segs = mlora.DeviceSegments(meta, W.n_rows, DEVICE)
    X = mlora.as_bf16_tensor(projs[0].X, DEVICE)
    Ys = [mlora.as_bf16_tensor(p.Y0, DEVICE) for p in projs]
    other = mlora.Pool(512, 256, 2, 8)          # another d_in
    cases = [([], []), ([pools[0], pools[0]], Ys), (pools, [Ys[0], Ys[0]]),
             ([pools[0], other], Ys), ([pools[0]] * 5, (Ys * 3)[:5])]
    for ps, ys in cases:
        with pytest.raises(mlora.MloraError) as e:
            mlora.apply_multi(ps, segs, X, ys)
        assert e.value.status == mlora.ERR_INVALID_ARG
    torch.cuda.synchronize()
    for p, Y in zip(projs, Ys):
        assert np.array_equal(mlora.bf16_bits(Y), p.Y0)
    other.close()
    free()


def test_fused_in_cuda_graph():
    W, projs = fused_case(47, 160, 1024, (1024, 256, 256), 5, (16,))
    pools = make_pools(W, projs)
    meta = mlora.build_segments(W.row_slot, pools[0])
    segs = mlora.DeviceSegments(meta, W.n_rows, DEVICE)
    X = mlora.as_bf16_tensor(projs[0].X, DEVICE)
    Y0 = [mlora.as_bf16_tensor(p.Y0, DEVICE) for p in projs]
    Ys = [y.clone() for y in Y0]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        mlora.apply_multi(pools, segs, X, Ys, stream=stream)   # warm-up (one-time set-up)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        mlora.apply_multi(pools, segs, X, Ys, stream=stream)
    for _ in range(3):
        for y, y0 in zip(Ys, Y0):
            y.copy_(y0)
        graph.replay()
    torch.cuda.synchronize()
    assert [pl.check() for pl in pools] == [0, 0, 0]
    check_all(W, projs, [mlora.bf16_bits(y) for y in Ys], "graph replay")
    del graph
    free()


def test_fused_full_size_block_attention_sampled():
    # the 70B-class attention inputs: q (8192 -> 8192), k and v (8192 -> 1024), 2048
    # decode rows over 128 rank-16 adapters, checked on sampled rows
    W = wl.make(5)
    W = dataclasses.replace(W, proj_shapes=W.proj_shapes[:3], _proj_cache={})
    projs = [W.projection(k) for k in range(3)]
    projs = [dataclasses.replace(p, X=projs[0].X) for p in projs]
    Ys, flags, _ = run_fused(W, projs)
    assert flags == [0, 0, 0]
    rows = sample_rows(W, 64)
    for k, (p, Y) in enumerate(zip(projs, Ys)):
        assert_close(Y[rows], oracle.reference(W, p, rows=rows), f"sampled rows, projection {k}")
    base = np.nonzero(W.row_slot < 0)[0]
    for p, Y in zip(projs, Ys):
        assert_untouched(Y, p.Y0, base, "base rows")
    free()


def test_fused_long_shrink_with_d_in_not_a_multiple_of_64():
    # one shrink launch for three projections whose d_in (200 = 3 x 64 + 8) ends inside a
    # 64-column block: each projection's A copy is cut at d_in, with a zeroed group after
    W, projs = fused_case(49, 900, 200, (256, 128, 384), 4, (8, 16, 64), base_frac=0.0, shuffle=False)
    assert mlora.build_segments(W.row_slot)["max_segment_rows"] >= 128
    Ys, flags, _ = run_fused(W, projs)
    assert flags == [0] * len(projs)
    check_all(W, projs, Ys, "long, d_in 200, 3 projections")
    free()
