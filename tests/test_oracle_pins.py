"""Pins for the fp64 oracle: facts the pages and the mathematics fix, independent of
the oracle's own code.

Each check below would fail under a plausible mistake in the oracle (a transposed
operand, a dropped scale or term, a wrong sign, a mis-scattered row); the mutant
test at the end plants such mistakes in a copy of the oracle and confirms it.

Sources (page title, section):
  * Multi-LoRA Serving: adapter batching -- "LoRA on one Linear layer"
    (Y = X W^T + s (X A^T) B^T, s = alpha/r, Delta W = s B A, P_LoRA = r(d_in+d_out)),
    "Why one adapter can be merged" (W'_a = W + s_a B_a A_a),
    "The math of a mixed batch" (base rows get X W^T only; rows keep their adapter),
    "What metadata a segmented kernel needs" (segment_offsets example, shrink/expand,
    scatter back with the same token -> adapter map).
  * S-LoRA deep dive -- section 1.1 (parameter count example), section 3.2
    (per-row gather formulation).
"""
import contextlib
import json
import os
import struct
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# helpers (inputs only; no oracle arithmetic is repeated here)
# ---------------------------------------------------------------------------

def _bf16(x):
    return wl.f32_to_bf16_bits(np.asarray(x, np.float32))


def _small_problem(seed=7, n_rows=24, d_in=40, d_out=48, n_slots=3, ranks=(2, 3, 5),
                   base_rows=(1, 5), shuffle=True):
    rng = np.random.default_rng(seed)
    slot_rank = np.array(ranks, np.int32)
    alpha = np.array([4.0, 6.0, 3.0][:n_slots])
    A = {s: _bf16(rng.normal(0, 0.3, (int(slot_rank[s]), d_in))) for s in range(n_slots)}
    B = {s: _bf16(rng.normal(0, 0.3, (d_out, int(slot_rank[s])))) for s in range(n_slots)}
    X = _bf16(rng.normal(0, 1, (n_rows, d_in)))
    Y0 = _bf16(rng.normal(0, 1, (n_rows, d_out)))
    row_slot = rng.integers(0, n_slots, n_rows).astype(np.int32)
    if not shuffle:
        row_slot = np.sort(row_slot)
    row_slot[list(base_rows)] = -1
    return dict(X=X, Y0=Y0, A=A, B=B, slot_rank=slot_rank, slot_alpha=alpha, row_slot=row_slot)


def _run_segments(P, meta=None, scales=None, Y0=None):
    meta = meta or _meta(P["row_slot"], P["slot_rank"])
    Y, flags = oracle.apply_segments(P["X"], P["Y0"] if Y0 is None else Y0, meta["offsets"],
                                     meta["slots"], meta["ranks"], scales,
                                     meta["token_indices"], P["slot_rank"], P["slot_alpha"],
                                     P["A"], P["B"])
    assert flags == 0
    return Y


def _meta(row_slot, slot_rank):
    off, slots, ti = oracle.group_rows(row_slot)
    ranks = np.array([0 if s < 0 else slot_rank[s] for s in slots], np.int32)
    return dict(offsets=off, slots=slots, ranks=ranks, token_indices=ti)


# ---------------------------------------------------------------------------
# pin checks (each returns normally or raises AssertionError)
# ---------------------------------------------------------------------------

def check_grouping_page_example():
    g = json.load(open(os.path.join(GOLDEN, "metadata_example.json")))
    off, slots, ti = oracle.group_rows(np.array(g["row_adapter"], np.int32))
    rank_of = {int(k): v for k, v in g["slot_rank"].items()}
    ranks = [0 if s < 0 else rank_of[int(s)] for s in slots]
    assert off.tolist() == g["expected"]["segment_offsets"]
    assert slots.tolist() == g["expected"]["adapter_slots"]
    assert ranks == g["expected"]["ranks"]
    assert ti.tolist() == g["expected"]["token_indices"]


def check_param_count_page_example():
    g = json.load(open(os.path.join(GOLDEN, "param_count.json")))
    n = oracle.adapter_params_read(g["d_in"], g["d_out"], g["r"])
    full = g["d_in"] * g["d_out"]
    assert int(n // 1000) / 10 == g["printed_lora_wan"]
    assert full // 10**4 == g["printed_full_wan"]
    assert full / n == g["printed_ratio"]
    for d_in, d_out, r in [(4096, 6144, 64), (8192, 1024, 16), (256, 256, 8), (14336, 4096, 32)]:
        assert oracle.adapter_params_read(d_in, d_out, r) == r * (d_in + d_out)


def check_merged_weight_identity(seed=3, d_in=16, d_out=24, r=2, n_rows=9):
    """Y0 = X W^T in fp64, then the oracle's branch must equal X (W + s B A)^T."""
    rng = np.random.default_rng(seed)
    X = _bf16(rng.normal(0, 1, (n_rows, d_in)))
    A = _bf16(rng.normal(0, 0.3, (r, d_in)))
    Bm = _bf16(rng.normal(0, 0.3, (d_out, r)))
    W = rng.normal(0, 0.1, (d_out, d_in))
    alpha = 5.0
    s = alpha / r
    Xd, Ad, Bd = oracle.bf16_to_f64(X), oracle.bf16_to_f64(A), oracle.bf16_to_f64(Bm)
    Y0 = Xd @ W.T
    row_slot = np.zeros(n_rows, np.int32)
    meta = _meta(row_slot, np.array([r], np.int32))
    Y, flags = oracle.apply_segments(X, Y0, meta["offsets"], meta["slots"], meta["ranks"], None,
                                     meta["token_indices"], np.array([r], np.int32),
                                     np.array([alpha]), {0: A}, {0: Bm})
    assert flags == 0
    merged = Xd @ (W + s * (Bd @ Ad)).T
    assert np.all(np.abs(Y - merged) <= 1e-12 * (1 + np.abs(merged)))


def check_zero_adapters_leave_y0():
    P = _small_problem()
    for which in ("A", "B"):
        Q = dict(P)
        Q[which] = {s: np.zeros_like(m) for s, m in P[which].items()}
        Y = _run_segments(Q)
        assert np.array_equal(Y, oracle.bf16_to_f64(P["Y0"]))


def check_base_rows_untouched():
    P = _small_problem()
    Y = _run_segments(P)
    base = P["row_slot"] < 0
    assert base.any()
    assert np.array_equal(Y[base], oracle.bf16_to_f64(P["Y0"][base]))
    assert not np.array_equal(Y[~base], oracle.bf16_to_f64(P["Y0"][~base]))


def check_row_permutation_invariance():
    P = _small_problem()
    Y = _run_segments(P)
    perm = np.random.default_rng(11).permutation(P["X"].shape[0])
    Q = dict(P, X=P["X"][perm], Y0=P["Y0"][perm], row_slot=P["row_slot"][perm])
    Yp = _run_segments(Q)
    assert np.array_equal(Yp, Y[perm])


def check_segment_split_invariance():
    P = _small_problem(shuffle=False)
    meta = _meta(P["row_slot"], P["slot_rank"])
    Y = _run_segments(P, meta)
    lens = np.diff(meta["offsets"])
    g = int(np.argmax(lens))
    assert lens[g] >= 2
    cut = int(meta["offsets"][g] + lens[g] // 2)
    off = np.insert(meta["offsets"], g + 1, cut)
    slots = np.insert(meta["slots"], g + 1, meta["slots"][g])
    ranks = np.insert(meta["ranks"], g + 1, meta["ranks"][g])
    Ys = _run_segments(P, dict(offsets=off, slots=slots, ranks=ranks,
                               token_indices=meta["token_indices"]))
    assert np.array_equal(Ys, Y)


def check_rank_zero_padding():
    P = _small_problem()
    meta = _meta(P["row_slot"], P["slot_rank"])
    scales = np.array([0.0 if s < 0 else P["slot_alpha"][s] / P["slot_rank"][s]
                       for s in meta["slots"]])
    Y = _run_segments(P, meta, scales=scales)
    pad = 64
    A = {s: np.vstack([m, np.zeros((pad - m.shape[0], m.shape[1]), np.uint16)])
         for s, m in P["A"].items()}
    B = {s: np.hstack([m, np.zeros((m.shape[0], pad - m.shape[1]), np.uint16)])
         for s, m in P["B"].items()}
    slot_rank = np.full_like(P["slot_rank"], pad)
    Q = dict(P, A=A, B=B, slot_rank=slot_rank)
    meta_q = dict(meta, ranks=np.where(meta["slots"] < 0, 0, pad).astype(np.int32))
    Yq = _run_segments(Q, meta_q, scales=scales)
    assert np.array_equal(Yq, Y)


def check_unit_vector_closed_form(i=5, j=7):
    """r = 1, A = e_i^T, B = e_j: row t gains s * X[t, i] in column j only."""
    P = _small_problem()
    d_in, d_out = P["X"].shape[1], P["Y0"].shape[1]
    one = _bf16([1.0])[0]
    A = np.zeros((1, d_in), np.uint16)
    A[0, i] = one
    Bm = np.zeros((d_out, 1), np.uint16)
    Bm[j, 0] = one
    n_slots = len(P["slot_rank"])
    Q = dict(P, A={s: A for s in range(n_slots)}, B={s: Bm for s in range(n_slots)},
             slot_rank=np.ones(n_slots, np.int32))
    Y = _run_segments(Q)
    Y0 = oracle.bf16_to_f64(P["Y0"])
    X = oracle.bf16_to_f64(P["X"])
    for t, a in enumerate(P["row_slot"].tolist()):
        expect = Y0[t].copy()
        if a >= 0:
            expect[j] = Y0[t, j] + P["slot_alpha"][a] / 1.0 * X[t, i]
        assert np.array_equal(Y[t], expect), t


def check_linearity():
    P = _small_problem()
    meta = _meta(P["row_slot"], P["slot_rank"])
    zero = np.zeros(P["Y0"].shape)
    sc = np.array([0.0 if s < 0 else 1.25 * (g + 1) for g, s in enumerate(meta["slots"])])
    Y1 = _run_segments(P, meta, scales=sc, Y0=zero)
    Y2 = _run_segments(P, meta, scales=2 * sc, Y0=zero)
    assert np.array_equal(Y2, 2 * Y1)
    # additivity in B over disjoint supports (so B1 + B2 is exact in bf16)
    B1 = {s: np.where(np.arange(m.shape[1])[None, :] % 2 == 0, m, 0).astype(np.uint16)
          for s, m in P["B"].items()}
    B2 = {s: np.where(np.arange(m.shape[1])[None, :] % 2 == 1, m, 0).astype(np.uint16)
          for s, m in P["B"].items()}
    Ya = _run_segments(dict(P, B=B1), meta, scales=sc, Y0=zero)
    Yb = _run_segments(dict(P, B=B2), meta, scales=sc, Y0=zero)
    assert np.all(np.abs(Y1 - (Ya + Yb)) <= 1e-12 * (1 + np.abs(Y1)))


def check_rows_equal_segments():
    P = _small_problem()
    Y = _run_segments(P)
    Yr, flags = oracle.apply_rows(P["X"], P["Y0"], P["row_slot"], None, P["slot_rank"],
                                  P["slot_alpha"], P["A"], P["B"])
    assert flags == 0
    assert np.array_equal(Y, Yr)


def _bf16_py(bits):
    return struct.unpack(">f", struct.pack(">I", int(bits) << 16))[0]


def check_brute_force_tiny():
    """Plain Python loops over the tiny workload, straight from the row formula."""
    W = wl.tiny()
    proj = W.projection(0)
    Y = oracle.reference(W, proj)
    n, d_in = proj.X.shape
    d_out = proj.Y0.shape[1]
    for t in range(n):
        a = int(W.row_slot[t])
        y0 = [_bf16_py(v) for v in proj.Y0[t]]
        if a < 0:
            assert Y[t].tolist() == y0
            continue
        r = int(W.slot_rank[a])
        s = W.slot_alpha[a] / r
        x = [_bf16_py(v) for v in proj.X[t]]
        Am = [[_bf16_py(v) for v in row] for row in proj.A[a]]
        Bm = [[_bf16_py(v) for v in row] for row in proj.B[a]]
        h = [sum(x[k] * Am[j][k] for k in range(d_in)) for j in range(r)]
        for o in range(d_out):
            want = y0[o] + s * sum(h[j] * Bm[o][j] for j in range(r))
            assert abs(Y[t, o] - want) <= 1e-12 * (1 + abs(want)), (t, o)


def check_shrink_expand_compose():
    P = _small_problem()
    meta = _meta(P["row_slot"], P["slot_rank"])
    Y = _run_segments(P, meta)
    H, f1 = oracle.shrink(P["X"], meta["offsets"], meta["slots"], meta["ranks"],
                          meta["token_indices"], P["slot_rank"], P["A"], 8,
                          H_init=np.zeros((P["X"].shape[0], 8)))
    Y2, f2 = oracle.expand(H, P["Y0"], meta["offsets"], meta["slots"], meta["ranks"], None,
                           meta["token_indices"], P["slot_rank"], P["slot_alpha"], P["B"])
    assert f1 == 0 and f2 == 0
    assert np.array_equal(Y2, Y)


def check_invalid_metadata_skipped():
    P = _small_problem()
    meta = _meta(P["row_slot"], P["slot_rank"])
    Y0 = oracle.bf16_to_f64(P["Y0"])
    g = int(np.nonzero(meta["slots"] >= 0)[0][0])
    rows = meta["token_indices"][meta["offsets"][g]:meta["offsets"][g + 1]]
    cases = [("slots", 99, oracle.BAD_SLOT), ("ranks", 77, oracle.BAD_RANK)]
    for key, val, flag in cases:
        bad = {k: v.copy() for k, v in meta.items()}
        bad[key][g] = val
        Y, flags = oracle.apply_segments(P["X"], P["Y0"], bad["offsets"], bad["slots"],
                                         bad["ranks"], None, bad["token_indices"],
                                         P["slot_rank"], P["slot_alpha"], P["A"], P["B"])
        assert flags & flag
        assert np.array_equal(Y[rows], Y0[rows])
    bad = {k: v.copy() for k, v in meta.items()}
    bad["token_indices"][meta["offsets"][g]] = 10**6
    Y, flags = oracle.apply_segments(P["X"], P["Y0"], bad["offsets"], bad["slots"], bad["ranks"],
                                     None, bad["token_indices"], P["slot_rank"],
                                     P["slot_alpha"], P["A"], P["B"])
    assert flags & oracle.BAD_ROW


PIN_CHECKS = [check_grouping_page_example, check_param_count_page_example,
              check_merged_weight_identity, check_zero_adapters_leave_y0,
              check_base_rows_untouched, check_row_permutation_invariance,
              check_segment_split_invariance, check_rank_zero_padding,
              check_unit_vector_closed_form, check_linearity, check_rows_equal_segments,
              check_brute_force_tiny, check_shrink_expand_compose,
              check_invalid_metadata_skipped]


@pytest.mark.parametrize("check", PIN_CHECKS, ids=[c.__name__ for c in PIN_CHECKS])
def test_pin(check):
    check()


def test_merged_weight_identity_tiny_workload():
    """The same identity at the tiny workload's size (d = 256, r = 8)."""
    check_merged_weight_identity(seed=0, d_in=256, d_out=256, r=8, n_rows=32)


def test_grouping_properties():
    rng = np.random.default_rng(5)
    for n in (0, 1, 7, 300):
        row_slot = rng.integers(-1, 9, n).astype(np.int32)
        off, slots, ti = oracle.group_rows(row_slot)
        assert off[0] == 0 and off[-1] == n and np.all(np.diff(off) > 0)
        assert sorted(ti.tolist()) == list(range(n))
        assert len(set(slots.tolist())) == len(slots)
        for g, s in enumerate(slots.tolist()):
            rows = ti[off[g]:off[g + 1]]
            assert np.all(row_slot[rows] == s)
            assert np.all(np.diff(rows) > 0)
        firsts = [int(ti[off[g]]) for g in range(len(slots))]
        assert firsts == sorted(firsts)


# ---------------------------------------------------------------------------
# planted mistakes: each mutant copy of the oracle must fail at least one pin
# ---------------------------------------------------------------------------

MUTANTS = {
    "transposed_B": ("bf16_value(b_row[j])", "bf16_value(B[(size_t)j * d_out + o])", 1),
    "dropped_scale": ("y[o] += s * acc;\n    }\n}", "y[o] += acc;\n    }\n}", 1),
    "wrong_sign": ("y[o] += s * acc;\n    }\n}", "y[o] -= s * acc;\n    }\n}", 1),
    "dropped_rank_term": ("for (int j = 0; j < r; ++j) acc += h[j]",
                          "for (int j = 1; j < r; ++j) acc += h[j]", None),
    "scale_alpha_times_r": ("slot_alpha[a] / (double)r", "slot_alpha[a] * (double)r", None),
    "scatter_to_grouped_position": ("int t = token_indices ? token_indices[p] : p;\n"
                                    "        if (t < 0 || t >= n_rows) { row_flags |= ORC_BAD_ROW; continue; }\n"
                                    "        double s",
                                    "int t = p;\n"
                                    "        if (t < 0 || t >= n_rows) { row_flags |= ORC_BAD_ROW; continue; }\n"
                                    "        double s", 1),
    "A_row_stride": ("A + (size_t)j * d_in;", "A + (size_t)j;", 1),
    "x_index": ("acc += bf16_value(x[k]) * bf16_value(a_row[k])",
                "acc += bf16_value(x[j]) * bf16_value(a_row[k])", 1),
    # the fp64-activation row (dtype boundary of a quantized base model)
    "xf64_x_index": ("dot += x[k] * bf16_value(arow_j[k])", "dot += x[j] * bf16_value(arow_j[k])", 1),
    "xf64_dropped_scale": ("y[o] = y[o] + s * dot;", "y[o] = y[o] + dot;", 1),
    "xf64_A_row_stride": ("A + (size_t)d_in * j;", "A + (size_t)j;", 1),
}


@contextlib.contextmanager
def _swapped_oracle(lib):
    saved = oracle._lib
    oracle._lib = lib
    try:
        yield
    finally:
        oracle._lib = saved


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    find, repl, count = MUTANTS[name]
    src = open(oracle._SRC).read()
    n = src.count(find)
    assert n >= 1 and (count is None or n == count), (name, n)
    mutated = src.replace(find, repl)
    cpath = tmp_path / "mutant.c"
    cpath.write_text(mutated)
    so = str(tmp_path / "libmutant.so")
    subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", so,
                    str(cpath)], check=True)
    lib = oracle.load(so)
    failed = []
    with _swapped_oracle(lib):
        for check in MUTANT_CHECKS:
            try:
                check()
            except AssertionError:
                failed.append(check.__name__)
    assert failed, f"mutant {name} passed every pin"


# ---------------------------------------------------------------------------
# the dtype boundary of a quantized base model: FP8 e4m3 activation codes and
# fp16 / fp32 base outputs (page "Multi-LoRA Serving: adapter batching", section
# "The dtype boundary between a quantized base model and LoRA")
# ---------------------------------------------------------------------------

def test_e4m3_decoding_closed_forms():
    # the format: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, subnormals at
    # exponent field 0, S.1111.111 NaN, no infinity
    v = oracle.e4m3_to_f64(np.array([0x38, 0x3C, 0x7E, 0x08, 0x01, 0x07, 0x00, 0xB8, 0xFE, 0x40], np.uint8))
    assert v.tolist() == [1.0, 1.5, 448.0, 2.0 ** -6, 2.0 ** -9, 7 * 2.0 ** -9, 0.0, -1.0, -448.0, 2.0]
    assert np.isnan(oracle.e4m3_to_f64(np.array([0x7F, 0xFF], np.uint8))).all()


def test_e4m3_decoding_matches_library_conversion():
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    both_nan = np.isnan(ours) & np.isnan(lib)
    assert np.array_equal(ours[~both_nan], lib[~both_nan]) and np.isnan(ours).sum() == np.isnan(lib).sum() == 2


def test_f16_decoding_closed_forms():
    v = oracle.f16_to_f64(np.array([0x3C00, 0x7BFF, 0x0001, 0xC000, 0x3555], np.uint16))
    assert v.tolist() == [1.0, 65504.0, 2.0 ** -24, -2.0, 0.333251953125]


def test_fp64_activation_entry_equals_bf16_entry():
    # the same activation values given as fp64 instead of bf16 bits: identical results
    P = _small_problem(seed=31)
    Yb, fb = oracle.apply_rows(P["X"], P["Y0"], P["row_slot"], None, P["slot_rank"], P["slot_alpha"],
                               P["A"], P["B"])
    Yx, fx = oracle.apply_rows_xf64(oracle.bf16_to_f64(P["X"]), oracle.bf16_to_f64(P["Y0"]), P["row_slot"],
                                    None, P["slot_rank"], P["slot_alpha"], P["A"], P["B"])
    assert fb == fx == 0
    assert np.array_equal(Yb, Yx)


def test_fp64_activation_merged_weight_identity_with_fp8_codes():
    # X = code * scale (FP8 activation), Y0 = X W^T in fp64: the result must equal
    # X (W + s B A)^T for adapter rows and X W^T for base rows
    rng = np.random.default_rng(5)
    P = _small_problem(seed=32, d_in=48, d_out=40)
    codes = rng.integers(0, 256, P["X"].shape).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38            # no NaN codes
    scale = 0.0625
    X = oracle.e4m3_to_f64(codes) * scale
    W = rng.normal(0, 0.5, (40, 48))
    Y0 = X @ W.T
    Y, flags = oracle.apply_rows_xf64(X, Y0, P["row_slot"], None, P["slot_rank"], P["slot_alpha"], P["A"], P["B"])
    assert flags == 0
    for t in range(X.shape[0]):
        a = int(P["row_slot"][t])
        Wt = W.copy()
        if a >= 0:
            s = P["slot_alpha"][a] / P["slot_rank"][a]
            Wt = W + s * oracle.bf16_to_f64(P["B"][a]) @ oracle.bf16_to_f64(P["A"][a])
        want = X[t] @ Wt.T
        assert np.allclose(Y[t], want, rtol=1e-12, atol=1e-12), t


def test_fp64_activation_is_linear_in_the_activation():
    # doubling X doubles the delta, exactly (powers of two scale fp64 sums exactly)
    P = _small_problem(seed=33)
    X = oracle.bf16_to_f64(P["X"])
    Y0 = np.zeros((X.shape[0], P["Y0"].shape[1]))
    Y1, _ = oracle.apply_rows_xf64(X, Y0, P["row_slot"], None, P["slot_rank"], P["slot_alpha"], P["A"], P["B"])
    Y2, _ = oracle.apply_rows_xf64(4 * X, Y0, P["row_slot"], None, P["slot_rank"], P["slot_alpha"], P["A"], P["B"])
    assert np.array_equal(Y2, 4 * Y1)
    assert np.abs(Y1).max() > 0


# the planted mistakes are judged by every pin, the fp64-activation ones included
MUTANT_CHECKS = PIN_CHECKS + [test_fp64_activation_entry_equals_bf16_entry,
                              test_fp64_activation_merged_weight_identity_with_fp8_codes,
                              test_fp64_activation_is_linear_in_the_activation]


# ---------------------------------------------------------------------------
# the base projection and the LoRA branch together (page "Multi-LoRA serving",
# ybb.press ai-applications, section 3.3: W0 x + B(A x) in one kernel)
# ---------------------------------------------------------------------------

def _base_problem(seed, n_rows, d_in, d_out, ranks, base_rows):
    rng = np.random.default_rng(seed)
    P = _small_problem(seed=seed, n_rows=n_rows, d_in=d_in, d_out=d_out, n_slots=len(ranks), ranks=ranks,
                       base_rows=base_rows)
    P["W"] = _bf16(rng.normal(0, 0.5, (d_out, d_in)))
    return P


def check_base_gemm_brute_force_tiny(fn=None):
    # every output element as explicit sums over k and over the rank, in Python floats
    fn = fn or oracle.base_gemm_apply
    P = _base_problem(41, n_rows=5, d_in=6, d_out=4, ranks=(2, 1), base_rows=(3,))
    Y, flags = fn(P["X"], P["W"], P["row_slot"], None, P["slot_rank"], P["slot_alpha"], P["A"], P["B"])
    assert flags == 0
    x, w = oracle.bf16_to_f64(P["X"]), oracle.bf16_to_f64(P["W"])
    for t in range(5):
        a = int(P["row_slot"][t])
        for o in range(4):
            want = sum(float(x[t, k]) * float(w[o, k]) for k in range(6))
            if a >= 0:
                r = int(P["slot_rank"][a])
                s = float(P["slot_alpha"][a]) / r
                av, bv = oracle.bf16_to_f64(P["A"][a]), oracle.bf16_to_f64(P["B"][a])
                for q in range(r):
                    h = sum(float(x[t, k]) * float(av[q, k]) for k in range(6))
                    want += s * h * float(bv[o, q])
            assert abs(Y[t, o] - want) <= 1e-12 * (1 + abs(want)), (t, o)


def check_base_gemm_merged_weight(fn=None):
    # adapter rows see the merged weight W + s B A, base rows W alone; square W, so a
    # missing transpose shows too
    fn = fn or oracle.base_gemm_apply
    P = _base_problem(42, n_rows=20, d_in=32, d_out=32, ranks=(3, 5, 2), base_rows=(0, 9))
    Y, flags = fn(P["X"], P["W"], P["row_slot"], None, P["slot_rank"], P["slot_alpha"], P["A"], P["B"])
    assert flags == 0
    x, w = oracle.bf16_to_f64(P["X"]), oracle.bf16_to_f64(P["W"])
    for t in range(20):
        a = int(P["row_slot"][t])
        Wt = w
        if a >= 0:
            s = P["slot_alpha"][a] / P["slot_rank"][a]
            Wt = w + s * oracle.bf16_to_f64(P["B"][a]) @ oracle.bf16_to_f64(P["A"][a])
        want = np.einsum("k,ok->o", x[t], Wt)
        assert np.allclose(Y[t], want, rtol=1e-12, atol=1e-12), t


def check_base_gemm_zero_weight_is_the_lora_branch(fn=None):
    # W = 0: exactly the LoRA branch onto a zero base output
    fn = fn or oracle.base_gemm_apply
    P = _base_problem(43, n_rows=16, d_in=24, d_out=20, ranks=(4, 2), base_rows=(2,))
    Z = np.zeros_like(P["W"])
    Y, _ = fn(P["X"], Z, P["row_slot"], None, P["slot_rank"], P["slot_alpha"], P["A"], P["B"])
    Yl, _ = oracle.apply_rows(P["X"], np.zeros((16, 20)), P["row_slot"], None, P["slot_rank"], P["slot_alpha"],
                              P["A"], P["B"])
    assert np.array_equal(Y, Yl) and np.all(Y[2] == 0)


BASE_GEMM_CHECKS = [check_base_gemm_brute_force_tiny, check_base_gemm_merged_weight,
                    check_base_gemm_zero_weight_is_the_lora_branch]


@pytest.mark.parametrize("check", BASE_GEMM_CHECKS, ids=[c.__name__ for c in BASE_GEMM_CHECKS])
def test_base_gemm_pin(check):
    check()


BASE_GEMM_MUTANTS = {
    "untransposed_W": ("bf16_to_f64(W).T", "bf16_to_f64(W)"),
    "dropped_base_term": ("return apply_rows(X, base,", "return apply_rows(X, 0 * base,"),
    "base_from_adapter_input": ("base = bf16_to_f64(X) @", "base = bf16_to_f64(X[::-1]) @"),
}


@pytest.mark.parametrize("name", sorted(BASE_GEMM_MUTANTS))
def test_base_gemm_planted_mistake_is_caught(name):
    import inspect
    find, repl = BASE_GEMM_MUTANTS[name]
    src = inspect.getsource(oracle.base_gemm_apply)
    assert src.count(find) == 1, name
    ns = dict(vars(oracle))
    exec(compile(src.replace(find, repl), "<mutant>", "exec"), ns)
    failed = []
    for check in BASE_GEMM_CHECKS:
        try:
            check(ns["base_gemm_apply"])
        except (AssertionError, ValueError):
            failed.append(check.__name__)
    assert failed, f"mutant {name} passed every pin"
