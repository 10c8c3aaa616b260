"""The seeded synthetic inputs follow their stated recipe: shapes, slot counts, ranks
and alphas of the five workloads, exact base-only counts, request lengths, the
bounded Zipf(1.1) slot draw, bf16 round-to-nearest-even, and determinism in the
seed.  (The inputs hold none of the method's arithmetic; these checks pin only how
they are drawn.)"""
import numpy as np
import pytest

import workloads as wl


def test_tiny_segments():
    W = wl.make(1)
    assert W.proj_shapes == [("proj", 256, 256)]
    assert W.n_slots == 4 and set(W.slot_rank.tolist()) == {8} and set(W.slot_alpha.tolist()) == {16.0}
    expect = np.concatenate([np.full(l, s) for l, s in zip([8, 4, 6, 9, 5], [0, -1, 1, 2, 3])])
    assert np.array_equal(W.row_slot, expect)


def test_qproj_decode_recipe():
    W = wl.make(2)
    assert W.proj_shapes == [("q_proj", 4096, 4096)]
    assert W.n_rows == 256 and W.n_slots == 64
    assert set(W.slot_rank.tolist()) == {16} and set(W.slot_alpha.tolist()) == {32.0}
    assert int((W.row_slot < 0).sum()) == round(0.10 * 256)
    assert W.row_slot.max() < 64


def test_qkv_prefill_recipe():
    W = wl.make(3)
    assert W.proj_shapes == [("qkv_proj", 4096, 6144)]
    assert W.n_slots == 8 and set(W.slot_rank.tolist()) == {64} and set(W.slot_alpha.tolist()) == {128.0}
    # eight requests, each a run of consecutive rows on its own slot
    change = np.nonzero(np.diff(W.row_slot))[0] + 1
    runs = np.split(W.row_slot, change)
    assert len(runs) == 8
    assert sorted(int(r[0]) for r in runs) == list(range(8))
    assert all(128 <= len(r) <= 2048 for r in runs)
    assert (W.row_slot >= 0).all()


def test_mixed_mlp_recipe():
    W = wl.make(4)
    assert W.proj_shapes == [("gate_proj", 4096, 14336), ("up_proj", 4096, 14336),
                             ("down_proj", 14336, 4096)]
    assert W.n_slots == 1024 and W.n_rows == 512 + 4 * 512
    assert set(W.slot_rank.tolist()) <= set(wl.RANK_BUCKETS)
    assert np.array_equal(W.slot_alpha, 2.0 * W.slot_rank)
    # the four prefill requests: runs of 512 rows on one slot each, after the decode rows
    for i in range(4):
        part = W.row_slot[512 + 512 * i:512 + 512 * (i + 1)]
        assert (part == part[0]).all()
    assert (W.row_slot >= 0).all()


def test_block70b_recipe():
    W = wl.make(5)
    assert [s[0] for s in W.proj_shapes] == ["q_proj", "k_proj", "v_proj", "o_proj", "gate_proj",
                                             "up_proj", "down_proj"]
    assert W.proj_shapes[1] == ("k_proj", 8192, 1024) and W.proj_shapes[6] == ("down_proj", 28672, 8192)
    assert W.n_rows == 2048 and W.n_slots == 128
    assert set(W.slot_rank.tolist()) == {16} and set(W.slot_alpha.tolist()) == {32.0}
    assert int((W.row_slot < 0).sum()) == round(0.05 * 2048)


def test_bounded_zipf_frequencies():
    rng = np.random.default_rng(123)
    n_slots, n = 64, 400_000
    draw = wl._zipf_slots(rng, n_slots, n)
    k = np.arange(1, n_slots + 1, dtype=np.float64)
    p = k ** -1.1 / (k ** -1.1).sum()
    freq = np.bincount(draw, minlength=n_slots) / n
    # within 5 standard errors for every slot
    se = np.sqrt(p * (1 - p) / n)
    assert np.all(np.abs(freq - p) < 5 * se + 1e-12)
    assert draw.min() >= 0 and draw.max() < n_slots


def test_bf16_round_to_nearest_even():
    one = np.float32(1.0)
    ulp = np.float32(2.0 ** -7)          # bf16 spacing at 1.0
    vals = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -20,
                     -(1.0 + 2.0 ** -8), 3.0e38], np.float32)
    got = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(vals))
    assert got[0] == one
    assert got[1] == one                 # tie, rounds to the even neighbour 1.0
    assert got[2] == one + 2 * ulp       # tie between 1+ulp and 1+2ulp: the even one
    assert got[3] == one + ulp           # above the tie: up
    assert got[4] == -one                # ties to even for negatives too
    assert np.isfinite(got[5])
    # exact for values that are already bf16
    x = wl.bf16_bits_to_f32(np.arange(0, 65536, 97, dtype=np.uint16))
    x = x[np.isfinite(x)]
    assert np.array_equal(wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(x)).view(np.uint32), x.view(np.uint32))


def test_deterministic_in_the_seed():
    a, b = wl.make(2), wl.make(2)
    assert np.array_equal(a.row_slot, b.row_slot)
    pa, pb = a.projection(0), b.projection(0)
    assert np.array_equal(pa.X, pb.X) and np.array_equal(pa.Y0, pb.Y0)
    assert all(np.array_equal(pa.A[s], pb.A[s]) and np.array_equal(pa.B[s], pb.B[s]) for s in pa.A)
    assert not np.array_equal(wl.qproj_decode(seed=7).row_slot, a.row_slot)


def test_value_distributions():
    p = wl.make(2).projection(0)
    X = wl.bf16_bits_to_f32(p.X)
    A = wl.bf16_bits_to_f32(np.concatenate([a.ravel() for a in p.A.values()]))
    assert abs(float(X.std()) - 1.0) < 0.01 and abs(float(X.mean())) < 0.01
    assert abs(float(A.std()) - wl.WEIGHT_STD) < 0.001
    # adapters exist exactly for the referenced slots, in the PEFT layout
    assert sorted(p.A) == sorted(wl.make(2).referenced_slots.tolist())
    s = next(iter(p.A))
    assert p.A[s].shape == (16, 4096) and p.B[s].shape == (4096, 16)


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_small_variants_keep_structure(cfg):
    full, small = wl.make(cfg), wl.make_small(cfg)
    assert small.proj_shapes == full.proj_shapes and small.n_slots == full.n_slots
    assert small.n_rows < full.n_rows
    lengths = np.bincount(small.row_slot[small.row_slot >= 0])
    lengths = lengths[lengths > 0]
    # segments that span several 8-row tiles and end on ragged tails
    assert lengths.max() > 8 and (lengths % 8 != 0).any()
