"""GPU edge cases through the C ABI: degenerate batches, every rank bucket and odd
ranks, ragged widths, partial coverage, strides, explicit scales, bad metadata,
standalone shrink / expand, pool reload and clear."""
import numpy as np
import pytest
import torch

import oracle
import segmented_rank_gemm_02_b200 as mlora
import workloads as wl
from gpu_harness import DEVICE, assert_close, assert_untouched, free, run_apply
from segmented_rank_gemm_02_b200 import staging

pytestmark = pytest.mark.gpu


def _ref(W, proj, meta, scales=None):
    Y, flags = oracle.apply_segments(proj.X, proj.Y0, meta["offsets"], meta["slots"],
                                     meta.get("ranks"), scales, meta.get("token_indices"),
                                     W.slot_rank, W.slot_alpha, proj.A, proj.B,
                                     n_tokens=meta.get("n_tokens"))
    return Y, flags


def _meta_from_oracle(W):
    off, slots, ti = oracle.group_rows(W.row_slot)
    ranks = np.array([0 if s < 0 else W.slot_rank[s] for s in slots], np.int32)
    return {"offsets": off, "slots": slots, "ranks": ranks, "token_indices": ti}


def test_empty_batch_is_noop():
    W = wl.random_case(1, 20, 64, 64, 3, (8,))
    proj = W.projection(0)
    meta = {"offsets": np.zeros(1, np.int32), "slots": np.zeros(0, np.int32),
            "token_indices": np.zeros(0, np.int32)}
    Y, flags, _ = run_apply(W, proj, meta=meta)
    assert flags == 0
    assert np.array_equal(Y, proj.Y0)


def test_all_base_rows_untouched():
    W = wl.random_case(2, 50, 128, 96, 3, (16,), base_frac=1.0)
    proj = W.projection(0)
    Y, flags, _ = run_apply(W, proj)
    assert flags == 0
    assert np.array_equal(Y, proj.Y0)


@pytest.mark.parametrize("d_in,d_out", [(264, 200), (1032, 72), (16, 8), (4096, 4096)])
def test_odd_ranks_and_ragged_widths(d_in, d_out):
    ranks = (1, 5, 8, 12, 16, 17, 31, 32, 33, 48, 63, 64)
    W = wl.random_case(3, 150, d_in, d_out, len(ranks), ranks, base_frac=0.15, r_max=64)
    W.slot_rank = np.array(ranks, np.int32)
    W.slot_alpha = 2.0 * W.slot_rank
    proj = W.projection(0)
    Y, flags, _ = run_apply(W, proj)
    assert flags == 0
    ref = oracle.reference(W, proj)
    assert_close(Y, ref, f"{d_in}x{d_out}")
    assert_untouched(Y, proj.Y0, np.nonzero(W.row_slot < 0)[0])


@pytest.mark.parametrize("r_max", [8, 16, 32, 64])
def test_every_pool_bucket(r_max):
    W = wl.random_case(4, 70, 512, 384, 5, (r_max,), base_frac=0.1)
    proj = W.projection(0)
    Y, flags, _ = run_apply(W, proj)
    assert flags == 0
    assert_close(Y, oracle.reference(W, proj), f"r_max={r_max}")


def test_length_one_segments_and_one_big_segment():
    # every row its own adapter (length-1 segments) ...
    W = wl.random_case(5, 64, 256, 256, 64, (16,), base_frac=0.0)
    W.row_slot = np.arange(64, dtype=np.int32)
    proj = W.projection(0)
    Y, flags, _ = run_apply(W, proj)
    assert flags == 0
    assert_close(Y, oracle.reference(W, proj), "length-1")
    # ... and one adapter over every row
    W.row_slot = np.full(64, 7, np.int32)
    proj = W.projection(0)
    Y, flags, _ = run_apply(W, proj)
    assert flags == 0
    assert_close(Y, oracle.reference(W, proj), "single segment")


def test_long_segments_consecutive_scattered_and_permuted():
    """Segments of >= 128 rows: consecutive rows (a prefill request: long-segment
    kernels, TMA tiles), rows scattered among another adapter's (decode-shaped kernel),
    and a permuted run of consecutive rows (long-segment kernels with row gathers)."""
    rng = np.random.default_rng(21)
    W = wl.random_case(21, 700, 512, 384, 3, (16, 64), base_frac=0.0, r_max=64)
    row_slot = np.empty(700, np.int32)
    row_slot[:260] = 0                       # rows 0..259: one request on slot 0
    row_slot[260:] = np.where(rng.random(440) < 0.5, 1, 2)   # slots 1, 2 interleaved
    W.row_slot = row_slot
    proj = W.projection(0)
    meta = _meta_from_oracle(W)
    assert int(np.diff(meta["offsets"]).min()) >= 128
    # permute the interior of the consecutive segment, keeping its first and last row
    ti = meta["token_indices"].copy()
    inner = ti[1:259].copy()
    rng.shuffle(inner)
    ti[1:259] = inner
    meta["token_indices"] = ti
    for name, m in (("consecutive + scattered", _meta_from_oracle(W)), ("permuted run", meta)):
        Y, flags, _ = run_apply(W, proj, meta=m)
        assert flags == 0
        ref, f = _ref(W, proj, m)
        assert f == 0
        assert_close(Y, ref, name)


def test_segment_mixing_scattered_rows_and_a_prefill_run():
    """One adapter's segment = its scattered decode rows, then a prefill request of
    consecutive rows (a mixed continuous batch): the chunks that are runs go to the
    long-segment kernels, the others to the decode-shaped kernel."""
    rng = np.random.default_rng(22)
    W = wl.random_case(22, 760, 512, 384, 3, (16, 32), base_frac=0.0, r_max=32)
    row_slot = np.empty(760, np.int32)
    row_slot[:300] = np.where(rng.random(300) < 0.5, 1, 2)   # decode rows, slots 1 and 2
    row_slot[300:] = 1                                       # a 460-row request on slot 1
    W.row_slot = row_slot
    proj = W.projection(0)
    meta = _meta_from_oracle(W)
    Y, flags, _ = run_apply(W, proj, meta=meta)
    assert flags == 0
    ref, f = _ref(W, proj, meta)
    assert f == 0
    assert_close(Y, ref, "mixed segment")


def test_apply_from_two_host_threads_on_one_pool():
    """Two host threads share a pool and a stream; their batches have long segments of
    different sizes, so the pool's workspace grows while the other thread launches."""
    import threading
    W = wl.random_case(23, 900, 512, 256, 2, (16,), base_frac=0.0, shuffle=False)
    proj = W.projection(0)
    pool = staging.make_pool(512, 256, W.n_slots, W.r_max, W.slot_rank, W.slot_alpha, proj.A, proj.B)
    stream = torch.cuda.Stream()
    ref = oracle.reference(W, proj)
    results, errors = {}, []

    def worker(n):
        try:
            meta = mlora.build_segments(W.row_slot[:n], pool)
            segs = mlora.DeviceSegments(meta, n, DEVICE)
            X = mlora.as_bf16_tensor(proj.X[:n], DEVICE)
            Y0 = mlora.as_bf16_tensor(proj.Y0[:n], DEVICE)
            Y = Y0.clone()
            torch.cuda.synchronize()
            for _ in range(5):
                with torch.cuda.stream(stream):
                    Y.copy_(Y0)
                    mlora.apply(pool, segs, X, Y, stream=stream)
            stream.synchronize()
            results[n] = mlora.bf16_bits(Y)
        except Exception as e:  # pragma: no cover
            errors.append(e)

    ts = [threading.Thread(target=worker, args=(n,)) for n in (300, 900)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors, errors
    assert pool.check() == 0
    for n, Y in results.items():
        # a prefix of the batch: each row gets the same delta as in the whole batch
        assert_close(Y, ref[:n], f"{n} rows")


def test_partial_coverage_and_empty_segments():
    W = wl.random_case(6, 90, 384, 256, 4, (16, 32), base_frac=0.0)
    proj = W.projection(0)
    meta = _meta_from_oracle(W)
    # drop the rows of the last segment from the metadata (they are uncovered) and add
    # two empty segments
    last = len(meta["slots"]) - 1
    n_tok = int(meta["offsets"][last])
    uncovered = meta["token_indices"][n_tok:]
    meta = {"offsets": np.concatenate([meta["offsets"][:last + 1], [n_tok, n_tok]]).astype(np.int32),
            "slots": np.concatenate([meta["slots"][:last], [1, 2]]).astype(np.int32),
            "ranks": np.concatenate([meta["ranks"][:last],
                                     [W.slot_rank[1], W.slot_rank[2]]]).astype(np.int32),
            "token_indices": meta["token_indices"][:n_tok].copy(), "n_tokens": n_tok}
    Y, flags, _ = run_apply(W, proj, meta=meta)
    assert flags == 0
    ref, f = _ref(W, proj, meta)
    assert f == 0
    assert_close(Y, ref, "partial")
    assert_untouched(Y, proj.Y0, uncovered)


def test_explicit_scales_and_no_ranks():
    W = wl.random_case(7, 80, 256, 320, 5, (8, 16, 32))
    proj = W.projection(0)
    meta = _meta_from_oracle(W)
    scales = np.array([0.0 if s < 0 else 0.37 * (g + 1) for g, s in enumerate(meta["slots"])],
                      np.float32)
    meta_nr = dict(meta)
    meta_nr.pop("ranks")
    Y, flags, _ = run_apply(W, proj, meta=meta_nr, scales=scales)
    assert flags == 0
    ref, f = _ref(W, proj, meta_nr, scales=scales.astype(np.float64))
    assert f == 0
    assert_close(Y, ref, "scales")


def test_identity_token_indices():
    W = wl.random_case(8, 100, 256, 256, 4, (16,), shuffle=False, base_frac=0.0)
    proj = W.projection(0)
    meta = _meta_from_oracle(W)
    assert np.array_equal(meta["token_indices"], np.arange(100))
    st = staging.upload(W, proj, DEVICE, meta=meta)
    segs = mlora.DeviceSegments(meta, W.n_rows, DEVICE, identity_rows=True)
    assert segs.token_indices is None
    mlora.apply(st["pool"], segs, st["X"], st["Y"])
    assert st["pool"].check() == 0
    assert_close(mlora.bf16_bits(st["Y"]), oracle.reference(W, proj), "identity")


def test_strided_inputs():
    W = wl.random_case(9, 60, 256, 128, 3, (16,))
    proj = W.projection(0)
    st = staging.upload(W, proj, DEVICE)
    Xw = torch.zeros(60, 256 + 64, dtype=torch.bfloat16, device=DEVICE)
    Yw = torch.zeros(60, 128 + 24, dtype=torch.bfloat16, device=DEVICE)
    Xw[:, :256] = st["X"]
    Yw[:, :128] = st["Y"]
    Xs, Ys = Xw[:, :256], Yw[:, :128]
    mlora.apply(st["pool"], st["segs"], Xs, Ys)
    assert st["pool"].check() == 0
    assert_close(mlora.bf16_bits(Ys.contiguous()), oracle.reference(W, proj), "strided")
    assert torch.count_nonzero(Yw[:, 128:]).item() == 0


@pytest.mark.parametrize("kind", ["slot", "rank", "row", "offsets", "empty_slot"])
def test_bad_metadata_is_flagged_and_skipped(kind):
    W = wl.random_case(10, 96, 256, 192, 4, (16,), base_frac=0.0)
    proj = W.projection(0)
    meta = _meta_from_oracle(W)
    g = 1
    p0, p1 = int(meta["offsets"][g]), int(meta["offsets"][g + 1])
    skipped = meta["token_indices"][p0:p1].copy()
    expect = {"slot": mlora.FLAG_BAD_SLOT, "rank": mlora.FLAG_BAD_RANK,
              "row": mlora.FLAG_BAD_ROW, "offsets": mlora.FLAG_BAD_OFFSETS,
              "empty_slot": mlora.FLAG_SLOT_EMPTY}[kind]
    meta = {k: v.copy() for k, v in meta.items()}
    st = staging.upload(W, proj, DEVICE)
    if kind == "slot":
        meta["slots"][g] = 1000
    elif kind == "rank":
        meta["ranks"][g] = 5
    elif kind == "row":
        meta["token_indices"][p0] = 10**6
        skipped = skipped[:1]
    elif kind == "offsets":
        # segment g claims positions past n_tokens; it is rejected, the others run
        meta["offsets"] = meta["offsets"].copy()
        meta["n_tokens"] = int(meta["offsets"][-1])
        meta["slots"] = np.concatenate([meta["slots"], [0]]).astype(np.int32)
        meta["ranks"] = np.concatenate([meta["ranks"], [W.slot_rank[0]]]).astype(np.int32)
        meta["offsets"] = np.concatenate([meta["offsets"], [meta["n_tokens"] + 5]]).astype(np.int32)
        skipped = np.zeros(0, np.int64)
    elif kind == "empty_slot":
        st["pool"].clear_slot(int(meta["slots"][g]))
    segs = mlora.DeviceSegments(meta, W.n_rows, DEVICE)
    mlora.apply(st["pool"], segs, st["X"], st["Y"])
    flags = st["pool"].check()
    assert flags & expect, (kind, flags)
    Y = mlora.bf16_bits(st["Y"])
    assert_untouched(Y, proj.Y0, skipped, kind)
    # every other adapter row still gets its delta
    slot_rank = W.slot_rank.copy()
    if kind == "empty_slot":
        slot_rank[int(meta["slots"][g])] = 0
    ref, f = oracle.apply_segments(proj.X, proj.Y0, meta["offsets"], meta["slots"],
                                   meta["ranks"], None, meta["token_indices"], slot_rank,
                                   W.slot_alpha, proj.A, proj.B, n_tokens=meta.get("n_tokens"))
    assert f & expect
    assert_close(Y, ref, kind)
    assert st["pool"].check() == 0   # cleared by the previous check


def _h_bound(W, proj, meta, r_cols):
    """Summation bound 2 (n + 16) u sum_k |x_k a_jk| for any order of fp32 additions
    (the factor 2 covers accumulators that truncate), from the oracle on |X| and |A|."""
    absX = proj.X & np.uint16(0x7FFF)
    absA = {s: m & np.uint16(0x7FFF) for s, m in proj.A.items()}
    S, _ = oracle.shrink(absX, meta["offsets"], meta["slots"], meta["ranks"],
                         meta["token_indices"], W.slot_rank, absA, r_cols)
    return 2.0 * (proj.d_in + 16) * 2.0 ** -24 * S + 1e-30


@pytest.mark.parametrize("cfg", [2, 4])
def test_shrink_matches_oracle(cfg):
    W = wl.make_small(cfg)
    proj = W.projection(0)
    st = staging.upload(W, proj, DEVICE)
    meta = st["meta"]
    r_cols = 64
    H = torch.full((st["segs"].n_tokens, r_cols), float("nan"), dtype=torch.float32, device=DEVICE)
    mlora.shrink(st["pool"], st["segs"], st["X"], H)
    assert st["pool"].check() == 0
    Hg = H.cpu().numpy().astype(np.float64)
    Href, f = oracle.shrink(proj.X, meta["offsets"], meta["slots"], meta["ranks"],
                            meta["token_indices"], W.slot_rank, proj.A, r_cols)
    assert f == 0
    bound = _h_bound(W, proj, meta, r_cols)
    written = ~np.isnan(Href)
    assert np.array_equal(~np.isnan(Hg), written)       # same entries written
    assert np.all(np.abs(Hg[written] - Href[written]) <= bound[written])


@pytest.mark.parametrize("cfg", [2, 4])
def test_expand_matches_oracle(cfg):
    W = wl.make_small(cfg)
    proj = W.projection(0)
    st = staging.upload(W, proj, DEVICE)
    meta = st["meta"]
    rng = np.random.default_rng(100 + cfg)
    Hh = rng.standard_normal((st["segs"].n_tokens, 64), dtype=np.float32)
    H = torch.from_numpy(Hh).to(DEVICE)
    mlora.expand(st["pool"], st["segs"], H, st["Y"])
    assert st["pool"].check() == 0
    ref, f = oracle.expand(Hh.astype(np.float64), proj.Y0, meta["offsets"], meta["slots"],
                           meta["ranks"], None, meta["token_indices"], W.slot_rank,
                           W.slot_alpha, proj.B)
    assert f == 0
    Y = mlora.bf16_bits(st["Y"])
    assert_close(Y, ref, "expand")
    assert_untouched(Y, proj.Y0, np.nonzero(W.row_slot < 0)[0])


def test_shrink_then_expand_equals_apply():
    W = wl.make_small(4)
    proj = W.projection(2)
    st = staging.upload(W, proj, DEVICE)
    H = torch.zeros((st["segs"].n_tokens, 64), dtype=torch.float32, device=DEVICE)
    mlora.shrink(st["pool"], st["segs"], st["X"], H)
    mlora.expand(st["pool"], st["segs"], H, st["Y"])
    assert st["pool"].check() == 0
    assert_close(mlora.bf16_bits(st["Y"]), oracle.reference(W, proj), "two-step")


def test_load_from_device_reload_and_clear():
    W = wl.random_case(11, 40, 256, 256, 3, (16,), base_frac=0.0)
    proj = W.projection(0)
    pool = mlora.Pool(256, 256, 3, 64)
    for s in proj.A:   # load from device tensors
        pool.load_slot(s, int(W.slot_rank[s]), float(W.slot_alpha[s]),
                       mlora.as_bf16_tensor(proj.A[s], DEVICE), mlora.as_bf16_tensor(proj.B[s], DEVICE))
    st = staging.upload(W, proj, DEVICE, pool=pool)
    mlora.apply(pool, st["segs"], st["X"], st["Y"])
    assert pool.check() == 0
    assert_close(mlora.bf16_bits(st["Y"]), oracle.reference(W, proj), "device load")
    # reload slot 0 with another rank and new weights; the result follows the new adapter
    rng = np.random.default_rng(12)
    r_new = 40
    A_new = wl.f32_to_bf16_bits(rng.normal(0, 0.02, (r_new, 256)).astype(np.float32))
    B_new = wl.f32_to_bf16_bits(rng.normal(0, 0.02, (256, r_new)).astype(np.float32))
    pool.load_slot(0, r_new, 80.0, A_new, B_new)
    assert pool.slot_info(0) == (r_new, 80.0, r_new * 512)
    W.slot_rank = W.slot_rank.copy()
    W.slot_alpha = W.slot_alpha.copy()
    W.slot_rank[0], W.slot_alpha[0] = r_new, 80.0
    proj.A[0], proj.B[0] = A_new, B_new
    st2 = staging.upload(W, proj, DEVICE, pool=pool)
    mlora.apply(pool, st2["segs"], st2["X"], st2["Y"])
    assert pool.check() == 0
    assert_close(mlora.bf16_bits(st2["Y"]), oracle.reference(W, proj), "reloaded")
    pool.clear_slot(0)
    assert pool.slot_info(0)[0] == 0
    pool.close()
    free()


def test_host_rejects_bad_arguments():
    W = wl.random_case(13, 16, 64, 64, 2, (8,))
    proj = W.projection(0)
    st = staging.upload(W, proj, DEVICE)
    pool = st["pool"]
    with pytest.raises(mlora.MloraError):
        pool.load_slot(5, 8, 16.0, proj.A[0], proj.B[0])          # slot out of range
    with pytest.raises(mlora.MloraError):
        pool.load_slot(0, 65, 16.0, proj.A[0], proj.B[0])         # rank above r_max
    Xbad = torch.zeros(16, 72, dtype=torch.bfloat16, device=DEVICE)[:, 1:65]   # misaligned
    with pytest.raises(mlora.MloraError):
        mlora.apply(pool, st["segs"], Xbad, st["Y"])
    Ynarrow = torch.zeros(16, 56, dtype=torch.bfloat16, device=DEVICE)   # row stride < d_out
    with pytest.raises(mlora.MloraError):
        mlora.apply(pool, st["segs"], st["X"], Ynarrow)


@pytest.mark.parametrize("d_in,ranks", [(200, (8, 64)), (4000, (16, 32)), (136, (64,))])
def test_long_segments_with_d_in_not_a_multiple_of_64(d_in, ranks):
    # prefill segments whose d_in ends inside a 64-column block: 200 = 3 x 64 + 8 (the
    # last tensor-core step half past d_in), 4000 = 62 x 64 + 32, 136 = 2 x 64 + 8; the
    # long-segment kernels take them, with rank buckets 8 to 64
    W = wl.random_case(90 + d_in, 900, d_in, 384, 4, ranks, base_frac=0.0, shuffle=False)
    proj = W.projection(0)
    meta = _meta_from_oracle(W)
    assert int(np.diff(meta["offsets"]).max()) >= 128
    Y, flags, _ = run_apply(W, proj, meta=meta)
    assert flags == 0
    ref, f = _ref(W, proj, meta)
    assert f == 0
    assert_close(Y, ref, f"d_in {d_in}")
    free()
