"""Slot lifecycle on the GPU: generations reject batches built for a replaced adapter,
a load from page-locked memory on one stream overlaps applies on another, and a
serving loop driven by the slot cache (loads on misses, evictions) stays exact."""
import numpy as np
import pytest
import torch

import oracle
import segmented_rank_gemm_02_b200 as mlora
import workloads as wl
from gpu_harness import DEVICE, assert_close, assert_untouched, free
from segmented_rank_gemm_02_b200 import staging

pytestmark = pytest.mark.gpu


def _meta(W, pool):
    m = mlora.build_segments(W.row_slot, pool)
    m["generations"] = np.array([0 if s < 0 else pool.generation(int(s)) for s in m["slots"]],
                                np.uint32)
    return m


def _ref(X, Y0, meta, slot_rank, slot_alpha, A, B):
    Y, flags = oracle.apply_segments(X, Y0, meta["offsets"], meta["slots"], meta.get("ranks"), None,
                                     meta["token_indices"], slot_rank, slot_alpha, A, B)
    assert flags == 0
    return Y


@pytest.mark.parametrize("n_rows,shuffle,base", [(96, True, 0.1), (600, False, 0.0)])
def test_stale_generation_is_rejected(n_rows, shuffle, base):
    # 600 sorted rows without base rows: segments of >= 128 consecutive rows (long kernels)
    W = wl.random_case(31, n_rows, 512, 384, 3, (16,), base_frac=base, shuffle=shuffle)
    proj = W.projection(0)
    pool = staging.make_pool(512, 384, W.n_slots, W.r_max, W.slot_rank, W.slot_alpha, proj.A, proj.B)
    meta = _meta(W, pool)
    assert all(pool.generation(s) == 1 for s in proj.A)
    # the batch as built: exact
    st = staging.upload(W, proj, DEVICE, pool=pool, meta=meta)
    mlora.apply(pool, st["segs"], st["X"], st["Y"])
    assert pool.check() == 0
    assert_close(mlora.bf16_bits(st["Y"]), oracle.reference(W, proj), "fresh")
    # slot 1 is reloaded (another adapter) after the batch was built: its rows are left alone
    rng = np.random.default_rng(5)
    A2 = wl.f32_to_bf16_bits(rng.standard_normal((16, 512), dtype=np.float32) * 0.02)
    B2 = wl.f32_to_bf16_bits(rng.standard_normal((384, 16), dtype=np.float32) * 0.02)
    pool.load_slot(1, 16, float(W.slot_alpha[1]), A2, B2)
    assert pool.generation(1) == 2
    st = staging.upload(W, proj, DEVICE, pool=pool, meta=meta)
    mlora.apply(pool, st["segs"], st["X"], st["Y"])
    assert pool.check() & mlora.FLAG_STALE_SLOT
    Y = mlora.bf16_bits(st["Y"])
    stale_rows = np.nonzero(W.row_slot == 1)[0]
    assert stale_rows.size > 0
    assert_untouched(Y, proj.Y0, stale_rows, "stale")
    ref = oracle.reference(W, proj)
    keep = np.nonzero((W.row_slot != 1))[0]
    assert_close(Y[keep], ref[keep], "other segments")
    # rebuilt with the new generation: slot 1 now applies adapter 2
    meta2 = _meta(W, pool)
    st = staging.upload(W, proj, DEVICE, pool=pool, meta=meta2)
    mlora.apply(pool, st["segs"], st["X"], st["Y"])
    assert pool.check() == 0
    A = dict(proj.A)
    B = dict(proj.B)
    A[1], B[1] = A2, B2
    assert_close(mlora.bf16_bits(st["Y"]), _ref(proj.X, proj.Y0, meta2, W.slot_rank, W.slot_alpha, A, B),
                 "rebuilt")
    # clearing advances the generation too
    pool.clear_slot(2)
    assert pool.generation(2) == 2
    del st
    free()


def test_load_on_one_stream_overlaps_apply_on_another():
    W = wl.random_case(32, 300, 1024, 768, 2, (32,), base_frac=0.0, shuffle=False)
    W.row_slot[:] = 0
    proj = W.projection(0)
    pool = mlora.Pool(1024, 768, 2, 32)
    pool.load_slot(0, 32, float(W.slot_alpha[0]), proj.A[0], proj.B[0])
    rng = np.random.default_rng(6)
    A1 = wl.f32_to_bf16_bits(rng.standard_normal((32, 1024), dtype=np.float32) * 0.02)
    B1 = wl.f32_to_bf16_bits(rng.standard_normal((768, 32), dtype=np.float32) * 0.02)
    A1p = torch.from_numpy(A1.view(np.int16)).pin_memory()
    B1p = torch.from_numpy(B1.view(np.int16)).pin_memory()
    torch.cuda.synchronize()
    s_apply, s_load = torch.cuda.Stream(), torch.cuda.Stream()
    meta0 = _meta(W, pool)
    st0 = staging.upload(W, proj, DEVICE, pool=pool, meta=meta0)
    Y1 = mlora.as_bf16_tensor(proj.Y0, DEVICE)
    torch.cuda.synchronize()
    # slot 1 loads from page-locked memory on s_load while s_apply applies slot 0
    mlora.apply(pool, st0["segs"], st0["X"], st0["Y"], stream=s_apply)
    pool.load_slot(1, 32, float(W.slot_alpha[1]), A1p, B1p, stream=s_load)
    loaded = torch.cuda.Event()
    loaded.record(s_load)
    assert pool.generation(1) == 1
    # then the same rows on slot 1, ordered after the load by the event
    row_slot1 = np.ones_like(W.row_slot)
    meta1 = mlora.build_segments(row_slot1, pool)
    meta1["generations"] = np.array([pool.generation(int(s)) for s in meta1["slots"]], np.uint32)
    segs1 = mlora.DeviceSegments(meta1, W.n_rows, DEVICE)
    s_apply.wait_event(loaded)
    mlora.apply(pool, segs1, st0["X"], Y1, stream=s_apply)
    torch.cuda.synchronize()
    assert pool.check() == 0
    A = {0: proj.A[0], 1: A1}
    B = {0: proj.B[0], 1: B1}
    ranks = np.array([32, 32], np.int32)
    assert_close(mlora.bf16_bits(st0["Y"]), _ref(proj.X, proj.Y0, meta0, ranks, W.slot_alpha, A, B), "slot 0")
    assert_close(mlora.bf16_bits(Y1), _ref(proj.X, proj.Y0, meta1, ranks, W.slot_alpha, A, B), "slot 1")
    free()


def test_serving_loop_with_the_slot_cache():
    """Batches over 6 adapters through a 3-slot pool: the cache pins each batch's slots,
    loads misses (evicting least recently used adapters), and every batch is exact."""
    d_in, d_out, n_slots = 512, 256, 3
    rng = np.random.default_rng(7)
    ranks = {a: int(r) for a, r in enumerate(rng.choice([8, 16, 32], size=6))}
    ad = {a: (wl.f32_to_bf16_bits(rng.standard_normal((ranks[a], d_in), dtype=np.float32) * 0.02),
              wl.f32_to_bf16_bits(rng.standard_normal((d_out, ranks[a]), dtype=np.float32) * 0.02))
          for a in ranks}
    alpha = {a: 2.0 * ranks[a] for a in ranks}
    pool = mlora.Pool(d_in, d_out, n_slots, 32)
    cache = mlora.SlotCache(n_slots)
    held = {}   # slot -> adapter
    for b in range(8):
        chosen = rng.choice(6, size=2, replace=False).tolist()
        n_rows = 40
        row_adapter = rng.choice(chosen, size=n_rows)
        slots = {}
        for a in chosen:
            s, needs_load, evicted = cache.acquire(int(a))
            if needs_load:
                pool.load_slot(s, ranks[a], alpha[a], ad[a][0], ad[a][1])
                held[s] = a
            assert held[s] == a
            slots[a] = s
        row_slot = np.array([slots[a] for a in row_adapter], np.int32)
        X = wl.f32_to_bf16_bits(rng.standard_normal((n_rows, d_in), dtype=np.float32))
        Y0 = wl.f32_to_bf16_bits(rng.standard_normal((n_rows, d_out), dtype=np.float32))
        meta = mlora.build_segments(row_slot, pool)
        meta["generations"] = np.array([pool.generation(int(s)) for s in meta["slots"]], np.uint32)
        segs = mlora.DeviceSegments(meta, n_rows, DEVICE)
        Xd = mlora.as_bf16_tensor(X, DEVICE)
        Yd = mlora.as_bf16_tensor(Y0, DEVICE)
        mlora.apply(pool, segs, Xd, Yd)
        assert pool.check() == 0
        slot_rank = np.zeros(n_slots, np.int32)
        slot_alpha = np.zeros(n_slots)
        A, B = {}, {}
        for s, a in held.items():
            slot_rank[s], slot_alpha[s] = ranks[a], alpha[a]
            A[s], B[s] = ad[a]
        assert_close(mlora.bf16_bits(Yd), _ref(X, Y0, meta, slot_rank, slot_alpha, A, B), f"batch {b}")
        for a in chosen:
            cache.release(slots[a])
    hits, misses, evictions = cache.stats()
    assert hits + misses == 16 and evictions == max(0, misses - n_slots)
    free()
