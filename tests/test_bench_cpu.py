"""Host-side pieces of the benchmark: which projections a fused step applies together,
and the algorithmic bytes a step moves (the roofline's numerator)."""
import numpy as np

import bench
import workloads as wl


def test_fusion_groups_of_the_workloads():
    assert bench.fusion_groups(wl.make_small(5), True) == [[0, 1, 2], [3], [4, 5], [6]]
    assert bench.fusion_groups(wl.make_small(4), True) == [[0, 1], [2]]
    assert bench.fusion_groups(wl.make_small(3), True) == [[0]]
    assert bench.fusion_groups(wl.make_small(5), False) == [[j] for j in range(7)]


def test_fusion_groups_need_a_common_input_width():
    W = wl.make_small(5)
    shapes = list(W.proj_shapes)
    shapes[1] = ("k_proj", 4096, 1024)   # k reads another input: not fused with q and v
    W.proj_shapes = shapes
    assert bench.fusion_groups(W, True) == [[0, 2], [1], [3], [4, 5], [6]]


def test_step_bytes_count_each_input_once_per_group():
    W = wl.make_small(5)
    n_l = int((W.row_slot >= 0).sum())
    plain = bench.workload_facts(W)
    fused = bench.workload_facts(W, bench.fusion_groups(W, True))
    # q/k/v share one X row read, gate/up another: three fewer X reads of width 8192
    assert plain["bytes"] - fused["bytes"] == 3 * n_l * 8192 * 2
    assert plain["flops"] == fused["flops"]
    # per projection: distinct adapters once, X once, Y read and written
    distinct = W.referenced_slots
    name, d_in, d_out = W.proj_shapes[0]
    w = sum(int(W.slot_rank[s]) * (d_in + d_out) * 2 for s in distinct)
    assert plain["per_projection"][0]["bytes"] == w + n_l * d_in * 2 + n_l * d_out * 4


def test_group_leaders():
    assert bench.group_leaders([[0, 1, 2], [3]]) == {0: 0, 1: 0, 2: 0, 3: 3}
    assert np.all(np.array(list(bench.group_leaders([[2], [0, 1]]).values())) == [2, 0, 0])
