"""CPU-only checks of the C ABI: the library loads without a GPU, exports every
function the header declares, rejects bad arguments on the host, and its host
grouping helper matches the oracle's grouping bit for bit."""
import ctypes
import json
import os
import re
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mlora.h")


@pytest.fixture(scope="module")
def mlora():
    from segmented_rank_gemm_02_b200 import build
    build.build()
    import segmented_rank_gemm_02_b200 as m
    m.lib()
    return m


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mlora_[a-z_]+)\s*\(", text)))


def test_header_functions_match_binding(mlora):
    assert _declared_functions() == sorted(mlora.EXPORTS)


def test_header_constants_match_binding(mlora):
    text = open(HEADER).read()
    defines = dict(re.findall(r"#define (MLORA_\w+)\s+(\d+)u?", text))
    assert int(defines["MLORA_MAX_FUSED"]) == mlora.MAX_FUSED
    for name in ("BAD_OFFSETS", "BAD_SLOT", "BAD_RANK", "BAD_ROW", "SLOT_EMPTY", "TIMEOUT", "STALE_SLOT"):
        assert int(defines["MLORA_FLAG_" + name]) == getattr(mlora, "FLAG_" + name)


def test_library_exports_every_declared_symbol(mlora):
    out = subprocess.run(["nm", "-D", "--defined-only", mlora.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (mlora_\w+)", out))
    missing = set(_declared_functions()) - exported
    assert not missing, missing
    for name in _declared_functions():
        assert hasattr(mlora.lib(), name)


def test_status_strings_and_version(mlora):
    for code in range(6):
        assert mlora.status_string(code)
    assert mlora.version() >= 100


def test_null_arguments_rejected_without_gpu(mlora):
    L = mlora.lib()
    seg = mlora.SegmentsStruct(0, 0, 0, 0, None, None, None, None, None)
    assert L.mlora_apply(None, ctypes.byref(seg), None, 0, None, 0, None) == mlora.ERR_INVALID_ARG
    assert L.mlora_shrink(None, ctypes.byref(seg), None, 0, None, 0, None) == mlora.ERR_INVALID_ARG
    assert L.mlora_expand(None, ctypes.byref(seg), None, 0, None, 0, None) == mlora.ERR_INVALID_ARG
    assert L.mlora_pool_load_slot(None, 0, 8, 16.0, None, None, 0, None) == mlora.ERR_INVALID_ARG
    assert L.mlora_pool_check(None, None, None) == mlora.ERR_INVALID_ARG
    assert L.mlora_pool_slot_info(None, 0, None, None, None) == mlora.ERR_INVALID_ARG
    assert L.mlora_pool_destroy(None) == mlora.OK
    # fused apply: no pool list, no pools, too many, or a null pool in the list
    null2 = (ctypes.c_void_p * 2)(None, None)
    lds = (ctypes.c_int64 * 2)(0, 0)
    assert L.mlora_apply_multi(None, 1, ctypes.byref(seg), None, 0, null2, lds, None) == mlora.ERR_INVALID_ARG
    for n in (0, mlora.MAX_FUSED + 1, 2):
        assert L.mlora_apply_multi(null2, n, ctypes.byref(seg), None, 0, null2, lds, None) == \
            mlora.ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert L.mlora_pool_create(0, 16, 1, 8, ctypes.byref(h)) == mlora.ERR_INVALID_ARG
    assert L.mlora_pool_create(12, 16, 1, 8, ctypes.byref(h)) == mlora.ERR_UNSUPPORTED
    assert L.mlora_pool_create(16, 16, 1, 65, ctypes.byref(h)) == mlora.ERR_UNSUPPORTED


def test_pool_create_without_device_fails_cleanly(mlora):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    h = ctypes.c_void_p()
    st = mlora.lib().mlora_pool_create(256, 256, 4, 8, ctypes.byref(h))
    assert st in (mlora.ERR_CUDA, mlora.ERR_UNSUPPORTED)
    assert h.value is None


def test_build_segments_page_example(mlora):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "metadata_example.json")))
    meta = mlora.build_segments(np.array(g["row_adapter"], np.int32))
    assert meta["offsets"].tolist() == g["expected"]["segment_offsets"]
    assert meta["slots"].tolist() == g["expected"]["adapter_slots"]
    assert meta["token_indices"].tolist() == g["expected"]["token_indices"]
    assert meta["max_segment_rows"] == 5


@pytest.mark.parametrize("seed,n,hi", [(0, 0, 4), (1, 1, 4), (2, 257, 9), (3, 4096, 1024),
                                       (4, 10000, 3)])
def test_build_segments_matches_oracle_grouping(mlora, seed, n, hi):
    rng = np.random.default_rng(seed)
    row_slot = rng.integers(-1, hi, n).astype(np.int32)
    meta = mlora.build_segments(row_slot)
    off, slots, ti = oracle.group_rows(row_slot)
    assert np.array_equal(meta["offsets"], off)
    assert np.array_equal(meta["slots"], slots)
    assert np.array_equal(meta["token_indices"], ti)
    # the hint: the longest adapter segment whose rows are consecutive, at least 1
    # (0 means "unknown" in mlora_segments)
    want = 1
    for g in range(len(slots)):
        a, b = off[g], off[g + 1]
        if slots[g] >= 0 and b > a and ti[b - 1] - ti[a] == b - a - 1:
            want = max(want, int(b - a))
    assert meta["max_segment_rows"] == want


def test_build_segments_workloads(mlora):
    import workloads as wl
    for cfg in (1, 2, 3, 4, 5):
        W = wl.make(cfg)
        meta = mlora.build_segments(W.row_slot)
        off, slots, ti = oracle.group_rows(W.row_slot)
        assert np.array_equal(meta["offsets"], off), cfg
        assert np.array_equal(meta["slots"], slots), cfg
        assert np.array_equal(meta["token_indices"], ti), cfg
