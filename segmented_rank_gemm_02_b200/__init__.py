"""Python binding of the mlora C ABI (include/mlora.h) -- argument marshalling only.

Every step of the LoRA branch runs in the CUDA kernels of ``libmlora.so``; this
module only turns PyTorch tensors and numpy arrays into pointers, sizes and
streams.  The library is loaded on first use; if it is missing, that first call
raises ImportError: there is no fallback path.

    import segmented_rank_gemm_02_b200 as mlora
    pool = mlora.Pool(d_in, d_out, n_slots, r_max)
    pool.load_slot(slot, rank, alpha, A, B)              # PEFT layout, bf16
    meta = mlora.build_segments(row_slots, pool)          # host grouping helper
    segs = mlora.DeviceSegments(meta, n_rows, device)     # device metadata
    mlora.apply(pool, segs, X, Y)                         # Y (= X W^T) += LoRA delta
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmlora.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_OUT_OF_MEMORY, ERR_BAD_METADATA, ERR_CUDA, ERR_NO_SLOT = range(7)
(FLAG_BAD_OFFSETS, FLAG_BAD_SLOT, FLAG_BAD_RANK, FLAG_BAD_ROW, FLAG_SLOT_EMPTY, FLAG_TIMEOUT,
 FLAG_STALE_SLOT) = (1, 2, 4, 8, 16, 32, 64)

# Every function the header declares (checked by the CPU test suite).
EXPORTS = ("mlora_pool_create", "mlora_pool_destroy", "mlora_pool_load_slot",
           "mlora_pool_clear_slot", "mlora_pool_slot_info", "mlora_pool_shape",
           "mlora_pool_check", "mlora_shrink", "mlora_expand", "mlora_apply",
           "mlora_apply_noalloc", "mlora_apply_multi", "mlora_apply_ex", "mlora_base_gemm_apply",
           "mlora_build_segments", "mlora_status_string",
           "mlora_version", "mlora_pool_slot_generation", "mlora_slot_cache_create",
           "mlora_slot_cache_destroy", "mlora_slot_cache_acquire", "mlora_slot_cache_release",
           "mlora_slot_cache_invalidate", "mlora_slot_cache_lookup", "mlora_slot_cache_stats")


class MloraError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class SegmentsStruct(ctypes.Structure):
    _fields_ = [("n_segments", ctypes.c_int32), ("n_rows", ctypes.c_int32),
                ("n_tokens", ctypes.c_int32), ("max_segment_rows", ctypes.c_int32),
                ("segment_offsets", ctypes.c_void_p), ("adapter_slots", ctypes.c_void_p),
                ("ranks", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("token_indices", ctypes.c_void_p), ("generations", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m segmented_rank_gemm_02_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    i32p = ctypes.POINTER(ctypes.c_int32)
    seg_p = ctypes.POINTER(SegmentsStruct)
    sig = {
        "mlora_pool_create": [i32, i32, i32, i32, ctypes.POINTER(vp)],
        "mlora_pool_destroy": [vp],
        "mlora_pool_load_slot": [vp, i32, i32, f32, vp, vp, i32, vp],
        "mlora_pool_clear_slot": [vp, i32, vp],
        "mlora_pool_slot_info": [vp, i32, i32p, ctypes.POINTER(f32), ctypes.POINTER(i64)],
        "mlora_pool_shape": [vp, i32p, i32p, i32p, i32p],
        "mlora_pool_check": [vp, vp, ctypes.POINTER(ctypes.c_uint32)],
        "mlora_shrink": [vp, seg_p, vp, i64, vp, i64, vp],
        "mlora_expand": [vp, seg_p, vp, i64, vp, i64, vp],
        "mlora_apply": [vp, seg_p, vp, i64, vp, i64, vp],
        "mlora_apply_noalloc": [vp, seg_p, vp, i64, vp, i64, vp],
        "mlora_apply_ex": [vp, seg_p, vp, i32, f32, i64, vp, i32, i64, vp],
        "mlora_base_gemm_apply": [vp, seg_p, vp, i64, vp, i64, vp, i64, vp],
        "mlora_apply_multi": [ctypes.POINTER(vp), i32, seg_p, vp, i64, ctypes.POINTER(vp),
                              ctypes.POINTER(i64), vp],
        "mlora_build_segments": [vp, i32, vp, vp, vp, i32p, i32p, vp, vp],
        "mlora_pool_slot_generation": [vp, i32, ctypes.POINTER(ctypes.c_uint32)],
        "mlora_slot_cache_create": [i32, ctypes.POINTER(vp)],
        "mlora_slot_cache_destroy": [vp],
        "mlora_slot_cache_acquire": [vp, ctypes.c_uint64, i32p, i32p, ctypes.POINTER(ctypes.c_uint64)],
        "mlora_slot_cache_release": [vp, i32],
        "mlora_slot_cache_invalidate": [vp, i32],
        "mlora_slot_cache_lookup": [vp, ctypes.c_uint64, i32p],
        "mlora_slot_cache_stats": [vp, ctypes.POINTER(i64), ctypes.POINTER(i64), ctypes.POINTER(i64)],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.mlora_status_string.argtypes = [ctypes.c_int]
    lib.mlora_status_string.restype = ctypes.c_char_p
    lib.mlora_version.argtypes = []
    lib.mlora_version.restype = ctypes.c_int32
    return lib


_lib_handle = None


def lib():
    """The loaded libmlora.so (loads it on first use; raises if it is not built)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load()
    return _lib_handle


def status_string(status: int) -> str:
    return lib().mlora_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != OK:
        raise MloraError(status, what)


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        return int(x.data_ptr())
    if isinstance(x, np.ndarray):
        return int(x.ctypes.data)
    return int(x)


def _ld(t, what: str) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{what} must be a 2-D row-major tensor")
    return int(t.stride(0))


def as_bf16_tensor(bits: np.ndarray, device=None):
    """bf16 bit patterns (numpy uint16) -> torch.bfloat16 tensor (bit-exact)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t if device is None else t.to(device)


def bf16_bits(t) -> np.ndarray:
    """torch.bfloat16 tensor -> numpy uint16 bit patterns."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class Pool:
    """A fixed-stride adapter pool for one projection (owns device memory)."""

    def __init__(self, d_in: int, d_out: int, n_slots: int, r_max: int):
        h = ctypes.c_void_p()
        _check(lib().mlora_pool_create(d_in, d_out, n_slots, r_max, ctypes.byref(h)),
               "mlora_pool_create")
        self.handle = h.value
        self.d_in, self.d_out, self.n_slots, self.r_max = d_in, d_out, n_slots, r_max

    def load_slot(self, slot: int, rank: int, alpha: float, A, B, stream=None) -> None:
        """A: bf16 [rank, d_in], B: bf16 [d_out, rank]; numpy uint16 bits or torch tensors."""
        keep = []

        def src(m):
            if isinstance(m, np.ndarray):
                m = np.ascontiguousarray(m, dtype=np.uint16)
                keep.append(m)
                return int(m.ctypes.data), 0
            m = m.contiguous()
            keep.append(m)
            return int(m.data_ptr()), int(m.is_cuda)

        pa, da = src(A)
        pb, db = src(B)
        if da != db:
            raise ValueError("A and B must both be host or both be device memory")
        _check(lib().mlora_pool_load_slot(self.handle, slot, rank, float(alpha), pa, pb, da,
                                         _stream_ptr(stream)), "mlora_pool_load_slot")
        if not da:
            # host sources are staged by the call itself; keep until it returns
            pass
        self._keep = keep

    def clear_slot(self, slot: int, stream=None) -> None:
        _check(lib().mlora_pool_clear_slot(self.handle, slot, _stream_ptr(stream)),
               "mlora_pool_clear_slot")

    def generation(self, slot: int) -> int:
        """Generation of the slot's contents (mlora_pool_slot_generation)."""
        g = ctypes.c_uint32()
        _check(lib().mlora_pool_slot_generation(self.handle, slot, ctypes.byref(g)),
               "mlora_pool_slot_generation")
        return int(g.value)

    def slot_info(self, slot: int):
        r, a, n = ctypes.c_int32(), ctypes.c_float(), ctypes.c_int64()
        _check(lib().mlora_pool_slot_info(self.handle, slot, ctypes.byref(r), ctypes.byref(a),
                                         ctypes.byref(n)), "mlora_pool_slot_info")
        return r.value, a.value, n.value

    def check(self, stream=None) -> int:
        """Synchronise, read and clear the device status word; returns the flag bits."""
        f = ctypes.c_uint32()
        st = lib().mlora_pool_check(self.handle, _stream_ptr(stream), ctypes.byref(f))
        if st not in (OK, ERR_BAD_METADATA):
            _check(st, "mlora_pool_check")
        return int(f.value)

    def close(self) -> None:
        if getattr(self, "handle", None):
            lib().mlora_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def build_segments(row_slots: np.ndarray, pool: Optional[Pool] = None) -> dict:
    """Host grouping helper (mlora_build_segments): numpy int32 arrays."""
    row_slots = np.ascontiguousarray(row_slots, dtype=np.int32)
    n = int(row_slots.shape[0])
    offsets = np.zeros(n + 1, np.int32)
    slots = np.zeros(max(n, 1), np.int32)
    ti = np.zeros(max(n, 1), np.int32)
    ranks = np.zeros(max(n, 1), np.int32)
    S, longest = ctypes.c_int32(), ctypes.c_int32()
    _check(lib().mlora_build_segments(_ptr(row_slots), n, _ptr(offsets), _ptr(slots), _ptr(ti),
                                     ctypes.byref(S), ctypes.byref(longest),
                                     pool.handle if pool is not None else None,
                                     _ptr(ranks) if pool is not None else None),
           "mlora_build_segments")
    S = S.value
    out = {"offsets": offsets[:S + 1].copy(), "slots": slots[:S].copy(),
           "token_indices": ti[:n].copy(), "max_segment_rows": longest.value}
    if pool is not None:
        out["ranks"] = ranks[:S].copy()
    return out


class DeviceSegments:
    """Segment metadata resident on the device, plus the C struct pointing at it."""

    def __init__(self, meta: dict, n_rows: int, device, scales=None, identity_rows=False,
                 generations=None):
        import torch
        dev = torch.device(device)
        self.offsets = torch.as_tensor(np.asarray(meta["offsets"], np.int32)).to(dev)
        self.slots = torch.as_tensor(np.asarray(meta["slots"], np.int32)).to(dev)
        r = meta.get("ranks")
        self.ranks = None if r is None else torch.as_tensor(np.asarray(r, np.int32)).to(dev)
        self.scales = None if scales is None else torch.as_tensor(
            np.asarray(scales, np.float32)).to(dev)
        ti = meta.get("token_indices")
        self.token_indices = (None if (ti is None or identity_rows)
                              else torch.as_tensor(np.asarray(ti, np.int32)).to(dev))
        n_tokens = int(meta.get("n_tokens", self.offsets[-1].item() if ti is None else len(ti)))
        gens = generations if generations is not None else meta.get("generations")
        self.generations = None if gens is None else torch.as_tensor(
            np.asarray(gens, np.uint32).view(np.int32)).to(dev)
        self.struct = SegmentsStruct(
            int(self.slots.numel()), int(n_rows), n_tokens, int(meta.get("max_segment_rows", 0)),
            _ptr(self.offsets), _ptr(self.slots), _ptr(self.ranks), _ptr(self.scales),
            _ptr(self.token_indices), _ptr(self.generations))

    @property
    def n_tokens(self) -> int:
        return int(self.struct.n_tokens)


def apply(pool: Pool, segs: DeviceSegments, X, Y, stream=None) -> None:
    """Y[t] = bf16(Y[t] + s (X[t] A^T) B^T) in place (mlora_apply)."""
    _check(lib().mlora_apply(pool.handle, ctypes.byref(segs.struct), _ptr(X), _ld(X, "X"),
                            _ptr(Y), _ld(Y, "Y"), _stream_ptr(stream)), "mlora_apply")


def apply_noalloc(pool: Pool, segs: DeviceSegments, X, Y, stream=None) -> None:
    """mlora_apply with the long-segment scratch in the library's fixed device array
    (mlora_apply_noalloc): allocates nothing; concurrent calls on the GPU race."""
    _check(lib().mlora_apply_noalloc(pool.handle, ctypes.byref(segs.struct), _ptr(X), _ld(X, "X"),
                                     _ptr(Y), _ld(Y, "Y"), _stream_ptr(stream)), "mlora_apply_noalloc")


MAX_FUSED = 4

DTYPE_BF16, DTYPE_FP16, DTYPE_FP32, DTYPE_FP8_E4M3 = 0, 1, 2, 3


def _dtype_code(t) -> int:
    import torch
    codes = {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_FP16, torch.float32: DTYPE_FP32,
             torch.float8_e4m3fn: DTYPE_FP8_E4M3}
    if t.dtype not in codes:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def apply_ex(pool: Pool, segs: DeviceSegments, X, Y, x_scale: float = 1.0, stream=None) -> None:
    """mlora_apply at a quantized base model's dtype boundary (mlora_apply_ex): X bf16 or
    FP8 e4m3 codes (value = code * x_scale), Y bf16, fp16 or fp32, updated in place."""
    _check(lib().mlora_apply_ex(pool.handle, ctypes.byref(segs.struct), _ptr(X), _dtype_code(X), float(x_scale),
                                _ld(X, "X"), _ptr(Y), _dtype_code(Y), _ld(Y, "Y"), _stream_ptr(stream)),
           "mlora_apply_ex")


def base_gemm_apply(pool: Pool, segs: DeviceSegments, X, W, Y, stream=None) -> None:
    """Y = bf16(X W^T + s (X A^T) B^T) for adapter rows, bf16(X W^T) for the others, in
    one pass (mlora_base_gemm_apply).  X [n_rows, d_in], W [d_out, d_in] (nn.Linear
    layout) and Y [n_rows, d_out], all bf16 on the pool's device; Y is written, not read."""
    _check(lib().mlora_base_gemm_apply(pool.handle, ctypes.byref(segs.struct), _ptr(X), _ld(X, "X"), _ptr(W),
                                       _ld(W, "W"), _ptr(Y), _ld(Y, "Y"), _stream_ptr(stream)),
           "mlora_base_gemm_apply")


def apply_multi(pools, segs: DeviceSegments, X, Ys, stream=None) -> None:
    """mlora_apply over several projections sharing X and the segments (q/k/v,
    gate/up): Ys[k] += delta of pools[k], in one pass over X (mlora_apply_multi)."""
    pools, Ys = list(pools), list(Ys)
    if len(pools) != len(Ys):
        raise ValueError("one output per pool")
    n = len(pools)
    handles = (ctypes.c_void_p * max(n, 1))(*[p.handle for p in pools])
    outs = (ctypes.c_void_p * max(n, 1))(*[_ptr(Y) for Y in Ys])
    lds = (ctypes.c_int64 * max(n, 1))(*[_ld(Y, "Y") for Y in Ys])
    _check(lib().mlora_apply_multi(handles, n, ctypes.byref(segs.struct), _ptr(X), _ld(X, "X"),
                                   outs, lds, _stream_ptr(stream)), "mlora_apply_multi")


def shrink(pool: Pool, segs: DeviceSegments, X, H, stream=None) -> None:
    """H[p, :r] = X[t_p] A^T, fp32, grouped order (mlora_shrink)."""
    _check(lib().mlora_shrink(pool.handle, ctypes.byref(segs.struct), _ptr(X), _ld(X, "X"),
                             _ptr(H), _ld(H, "H"), _stream_ptr(stream)), "mlora_shrink")


def expand(pool: Pool, segs: DeviceSegments, H, Y, stream=None) -> None:
    """Y[t_p] = bf16(Y[t_p] + s H[p, :r] B^T) in place (mlora_expand)."""
    _check(lib().mlora_expand(pool.handle, ctypes.byref(segs.struct), _ptr(H), _ld(H, "H"),
                             _ptr(Y), _ld(Y, "Y"), _stream_ptr(stream)), "mlora_expand")


class SlotCache:
    """Host-side adapter cache over a pool's slots (mlora_slot_cache): LRU order among
    unpinned slots, pin counts for in-flight batches.  Needs no GPU."""

    NONE = 2 ** 64 - 1

    def __init__(self, n_slots: int):
        h = ctypes.c_void_p()
        _check(lib().mlora_slot_cache_create(int(n_slots), ctypes.byref(h)), "mlora_slot_cache_create")
        self.handle = h.value

    def acquire(self, adapter_id: int):
        """(slot, needs_load, evicted_id or None); pins the slot."""
        s, nl, ev = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_uint64()
        _check(lib().mlora_slot_cache_acquire(self.handle, ctypes.c_uint64(adapter_id), ctypes.byref(s),
                                             ctypes.byref(nl), ctypes.byref(ev)),
               "mlora_slot_cache_acquire")
        return s.value, bool(nl.value), (None if ev.value == self.NONE else int(ev.value))

    def release(self, slot: int) -> None:
        _check(lib().mlora_slot_cache_release(self.handle, int(slot)), "mlora_slot_cache_release")

    def invalidate(self, slot: int) -> None:
        _check(lib().mlora_slot_cache_invalidate(self.handle, int(slot)), "mlora_slot_cache_invalidate")

    def lookup(self, adapter_id: int) -> int:
        s = ctypes.c_int32()
        _check(lib().mlora_slot_cache_lookup(self.handle, ctypes.c_uint64(adapter_id), ctypes.byref(s)),
               "mlora_slot_cache_lookup")
        return s.value

    def stats(self):
        h, m, e = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(lib().mlora_slot_cache_stats(self.handle, ctypes.byref(h), ctypes.byref(m), ctypes.byref(e)),
               "mlora_slot_cache_stats")
        return h.value, m.value, e.value

    def close(self) -> None:
        if getattr(self, "handle", None):
            lib().mlora_slot_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def version() -> int:
    return int(lib().mlora_version())
