"""ctypes binding of libkvpaged.so (include/kvpaged.h), argument marshalling only.

Every function keeps the C name. Device arguments are torch CUDA tensors
(their data pointers are passed through); host arrays are numpy arrays. All
computation happens in the library; there is no fallback: if the library has
not been built, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvpaged.so")

KV_OK = 0
KV_ERR_ARG = -1
KV_ERR_OOM = -2
KV_ERR_BAD_ID = -3
KV_ERR_DOUBLE_FREE = -4
KV_ERR_SHARED_TAIL = -5
KV_ERR_CUDA = -6
KV_ERR_WORKSPACE = -7
KV_ERR_UNSUPPORTED = -8
STATUS_NAMES = {0: "OK", -1: "ARG", -2: "OOM", -3: "BAD_ID", -4: "DOUBLE_FREE", -5: "SHARED_TAIL", -6: "CUDA",
                -7: "WORKSPACE", -8: "UNSUPPORTED"}

KV_DTYPE_F32, KV_DTYPE_BF16, KV_DTYPE_F16, KV_DTYPE_FP8_E4M3 = 0, 1, 2, 3
DTYPE_CODE = {"fp32": 0, "bf16": 1, "fp16": 2, "e4m3": 3}  # K/V pool types (e4m3: launch queries only)

KV_DEV_ERR_PAGE_RANGE = 1
KV_DEV_ERR_SEQ_LEN = 2
KV_DEV_ERR_SLOT = 4
KV_DEV_ERR_TIMEOUT = 8
KV_DEV_ERR_PIPELINE = 16
KV_DEV_ERR_POSITION = 32

# (name, restype, argtypes) of every exported function.
_i32, _i64, _u64, _vp, _f32, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t
_pi32 = ctypes.POINTER(ctypes.c_int32)
_pi64 = ctypes.POINTER(ctypes.c_int64)
_psz = ctypes.POINTER(ctypes.c_size_t)
_pvp = ctypes.POINTER(ctypes.c_void_p)
SIGNATURES = [
    ("kv_status_string", ctypes.c_char_p, [ctypes.c_int]),
    ("kv_version", ctypes.c_int, []),
    ("kv_pool_create", ctypes.c_int, [_i32, _i32, _vp, _pvp]),
    ("kv_pool_destroy", ctypes.c_int, [_vp]),
    ("kv_pool_alloc", ctypes.c_int, [_vp, _i32, _vp]),
    ("kv_pool_free", ctypes.c_int, [_vp, _i32, _vp]),
    ("kv_pool_incref", ctypes.c_int, [_vp, _i32, _vp]),
    ("kv_pool_refcount", ctypes.c_int, [_vp, _i32, _pi32]),
    ("kv_pool_num_free", ctypes.c_int, [_vp, _pi32]),
    ("kv_pool_page_size", ctypes.c_int, [_vp, _pi32]),
    ("kv_blocks_for_len", ctypes.c_int, [_i32, _i32, _pi32, _pi32, _pi32]),
    ("kv_cache_bytes", ctypes.c_int, [_i64, _i64, _i64, _i64, _i64, _i64, _pi64]),
    ("kv_slot_for_pos", ctypes.c_int, [_vp, _i32, _i32, _i64, _pi64]),
    ("kv_slots_for_range", ctypes.c_int, [_vp, _i32, _i32, _i64, _i64, _vp]),
    ("kv_append_slots", ctypes.c_int, [_vp, _i32, _vp, _i32, _vp, _vp]),
    ("kv_pool_cow_tails", ctypes.c_int, [_vp, _i32, _vp, _i32, _vp, _vp, _vp, _pi32]),
    ("kv_copy_pages", ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    ("kv_prefix_index_create", ctypes.c_int, [_i32, _u64, _pvp]),
    ("kv_prefix_index_destroy", ctypes.c_int, [_vp]),
    ("kv_prefix_register", ctypes.c_int, [_vp, _vp, _vp, _i32, _vp]),
    ("kv_prefix_match", ctypes.c_int, [_vp, _vp, _i32, _i32, _vp, _pi32]),
    ("kv_prefix_num_entries", ctypes.c_int, [_vp, _pi32]),
    ("kv_append", ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    ("kv_rope_append", ctypes.c_int,
     [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    ("paged_decode_attention", ctypes.c_int,
     [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _i32, _vp, _sz, _vp, _vp]),
    ("paged_decode_attention_append", ctypes.c_int,
     [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _i32, _vp, _sz, _vp,
      _vp]),
    ("paged_decode_attention_noalloc", ctypes.c_int,
     [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _i32, _vp, _vp]),
    ("kv_append_fp8", ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    ("paged_decode_attention_fp8", ctypes.c_int,
     [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp,
      _vp]),
    ("paged_decode_attention_rope_append", ctypes.c_int,
     [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32,
      _i32, _vp, _sz, _vp, _vp]),
    ("paged_prefill_attention", ctypes.c_int,
     [_vp, _vp, _vp, _i32, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp]),
    ("paged_decode_set_kernel", ctypes.c_int, [_i32]),
    ("paged_decode_num_splits", ctypes.c_int, [_i32, _i32, _i32, _i32, _i32, _pi32]),
    ("paged_decode_launch_info", ctypes.c_int, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _pi32, _pi32]),
    ("paged_decode_workspace_bytes", ctypes.c_int, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, _psz]),
]

_LIB = None


class KvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        self.name = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{fn} failed: KV_ERR_{self.name} ({status})")


def lib() -> ctypes.CDLL:
    """Load libkvpaged.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_433_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def _check(fn: str, rc: int) -> None:
    if rc != KV_OK:
        raise KvError(fn, rc)


def _np_i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


# ---------------------------------------------------------------- host helpers
def kv_blocks_for_len(length: int, page_size: int):
    a, b, c = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check("kv_blocks_for_len", lib().kv_blocks_for_len(length, page_size, a, b, c))
    return a.value, b.value, c.value


def kv_cache_bytes(L: int, B: int, T: int, H_kv: int, Dh: int, bytes_per_elem: int) -> int:
    out = ctypes.c_int64()
    _check("kv_cache_bytes", lib().kv_cache_bytes(L, B, T, H_kv, Dh, bytes_per_elem, out))
    return out.value


def kv_slot_for_pos(table_row: Sequence[int], page_size: int, pos: int) -> int:
    row = _np_i32(table_row)
    out = ctypes.c_int64()
    _check("kv_slot_for_pos", lib().kv_slot_for_pos(_p(row), row.size, page_size, pos, out))
    return out.value


def kv_slots_for_range(table_row: Sequence[int], page_size: int, start: int, n: int) -> np.ndarray:
    row = _np_i32(table_row)
    out = np.empty(n, dtype=np.int64)
    _check("kv_slots_for_range", lib().kv_slots_for_range(_p(row), row.size, page_size, start, n, _p(out)))
    return out


class KvPool:
    """Refcounted physical page pool (kv_pool_*)."""

    def __init__(self, num_pages: int, page_size: int, init_free_order: Optional[Sequence[int]] = None):
        self._h = ctypes.c_void_p()
        order = None if init_free_order is None else _np_i32(init_free_order)
        if order is not None and order.size != num_pages:
            raise KvError("kv_pool_create", KV_ERR_ARG)
        _check("kv_pool_create", lib().kv_pool_create(num_pages, page_size, _p(order), ctypes.byref(self._h)))
        self.num_pages = num_pages
        self.page_size = page_size

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h:
            lib().kv_pool_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def alloc(self, n: int) -> np.ndarray:
        out = np.empty(max(n, 0), dtype=np.int32)
        _check("kv_pool_alloc", lib().kv_pool_alloc(self._h, n, _p(out)))
        return out

    def free(self, ids) -> None:
        a = _np_i32(ids)
        _check("kv_pool_free", lib().kv_pool_free(self._h, a.size, _p(a)))

    def incref(self, ids) -> None:
        a = _np_i32(ids)
        _check("kv_pool_incref", lib().kv_pool_incref(self._h, a.size, _p(a)))

    def refcount(self, page: int) -> int:
        out = ctypes.c_int32()
        _check("kv_pool_refcount", lib().kv_pool_refcount(self._h, page, out))
        return out.value

    def num_free(self) -> int:
        out = ctypes.c_int32()
        _check("kv_pool_num_free", lib().kv_pool_num_free(self._h, out))
        return out.value

    def append_slots(self, block_tables: np.ndarray, seq_lens: np.ndarray) -> np.ndarray:
        """kv_append_slots on host arrays (int32 [B, max_blocks] and int32 [B], updated in place)."""
        assert block_tables.dtype == np.int32 and block_tables.flags.c_contiguous
        assert seq_lens.dtype == np.int32 and seq_lens.flags.c_contiguous
        B = seq_lens.size
        slots = np.empty(B, dtype=np.int64)
        _check("kv_append_slots", lib().kv_append_slots(self._h, B, _p(block_tables), block_tables.shape[1],
                                                         _p(seq_lens), _p(slots)))
        return slots


    def cow_tails(self, block_tables: np.ndarray, seq_lens: np.ndarray):
        """kv_pool_cow_tails on host arrays (table updated in place); returns (src, dst) int32 arrays."""
        assert block_tables.dtype == np.int32 and block_tables.flags.c_contiguous
        lens = _np_i32(seq_lens)
        B = lens.size
        src = np.empty(max(B, 1), dtype=np.int32)
        dst = np.empty(max(B, 1), dtype=np.int32)
        n = ctypes.c_int32()
        _check("kv_pool_cow_tails", lib().kv_pool_cow_tails(self._h, B, _p(block_tables), block_tables.shape[1], _p(lens),
                                                             _p(src), _p(dst), n))
        return src[: n.value].copy(), dst[: n.value].copy()


class KvPrefixIndex:
    """Chained-hash prefix index over full pages (kv_prefix_*)."""

    def __init__(self, page_size: int, salt: int = 0):
        self._h = ctypes.c_void_p()
        _check("kv_prefix_index_create", lib().kv_prefix_index_create(page_size, salt, ctypes.byref(self._h)))
        self.page_size = page_size

    def close(self):
        if self._h:
            lib().kv_prefix_index_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def register(self, pool: KvPool, tokens, page_ids) -> None:
        t = _np_i32(tokens)
        p = _np_i32(page_ids)
        if p.size < t.size // self.page_size:
            raise KvError("kv_prefix_register", KV_ERR_ARG)
        _check("kv_prefix_register", lib().kv_prefix_register(self._h, pool.handle, _p(t), t.size, _p(p)))

    def match(self, tokens) -> np.ndarray:
        t = _np_i32(tokens)
        out = np.empty(max(t.size // self.page_size, 1), dtype=np.int32)
        n = ctypes.c_int32()
        _check("kv_prefix_match", lib().kv_prefix_match(self._h, _p(t), t.size, self.page_size, _p(out), n))
        return out[: n.value].copy()

    def num_entries(self) -> int:
        n = ctypes.c_int32()
        _check("kv_prefix_num_entries", lib().kv_prefix_num_entries(self._h, n))
        return n.value


# ---------------------------------------------------------------- device calls
def _torch_dtype_code(t) -> int:
    import torch

    m = {torch.float32: KV_DTYPE_F32, torch.bfloat16: KV_DTYPE_BF16, torch.float16: KV_DTYPE_F16,
         torch.uint8: KV_DTYPE_FP8_E4M3}
    if t.dtype not in m:
        raise KvError("dtype", KV_ERR_ARG)
    return m[t.dtype]


def _stream(stream) -> Optional[int]:
    import torch

    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dev(t, name: str, dtype=None):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    return t.data_ptr()


def kv_append(k_pages, v_pages, k_new, v_new, slot_mapping, page_size: int, err_flag=None, stream=None) -> None:
    """k/v_pages [num_pages, H_kv, P, Dh]; k/v_new [B, H_kv, Dh]; slot_mapping int64 [B] (device)."""
    import torch

    num_pages, H_kv, P, Dh = k_pages.shape
    assert P == page_size and v_pages.shape == k_pages.shape
    B = k_new.shape[0]
    assert tuple(k_new.shape) == (B, H_kv, Dh) and v_new.shape == k_new.shape
    dt = _torch_dtype_code(k_pages)
    rc = lib().kv_append(_dev(k_pages, "k_pages"), _dev(v_pages, "v_pages", k_pages.dtype), _dev(k_new, "k_new", k_pages.dtype),
                         _dev(v_new, "v_new", k_pages.dtype), _dev(slot_mapping, "slot_mapping", torch.int64), B, H_kv, Dh,
                         page_size, num_pages, dt, _dev(err_flag, "err_flag", torch.int32), _stream(stream))
    _check("kv_append", rc)


KV_ROPE_HALF, KV_ROPE_INTERLEAVED = 0, 1
ROPE_STYLE = {"half": KV_ROPE_HALF, "interleaved": KV_ROPE_INTERLEAVED}


def kv_rope_append(k_pages, v_pages, k_new, v_new, slot_mapping, positions, cos_sin, page_size: int,
                   style: str = "half", q=None, q_out=None, err_flag=None, stream=None) -> None:
    """Rotate k_new (and q, into q_out; q_out may be q) by `positions`, then append.

    k/v_pages [num_pages, H_kv, P, Dh]; k/v_new [B, H_kv, Dh]; q/q_out [B, H_q, Dh];
    slot_mapping int64 [B]; positions int32 [B]; cos_sin fp32 [max_pos, Dh] (all device)."""
    import torch

    num_pages, H_kv, P, Dh = k_pages.shape
    assert P == page_size and v_pages.shape == k_pages.shape
    B = k_new.shape[0]
    assert tuple(k_new.shape) == (B, H_kv, Dh) and v_new.shape == k_new.shape
    assert cos_sin.dim() == 2 and cos_sin.shape[1] == Dh
    H_q = 0
    if q is not None:
        assert q_out is not None and q.shape == q_out.shape and q.shape[0] == B and q.shape[2] == Dh
        H_q = q.shape[1]
    dt = _torch_dtype_code(k_pages)
    rc = lib().kv_rope_append(_dev(k_pages, "k_pages"), _dev(v_pages, "v_pages", k_pages.dtype),
                              _dev(q_out, "q_out", k_pages.dtype), _dev(q, "q", k_pages.dtype),
                              _dev(k_new, "k_new", k_pages.dtype), _dev(v_new, "v_new", k_pages.dtype),
                              _dev(slot_mapping, "slot_mapping", torch.int64), _dev(positions, "positions", torch.int32),
                              _dev(cos_sin, "cos_sin", torch.float32), cos_sin.shape[0], ROPE_STYLE[style], B, H_q, H_kv,
                              Dh, page_size, num_pages, dt, _dev(err_flag, "err_flag", torch.int32), _stream(stream))
    _check("kv_rope_append", rc)


def kv_append_fp8(k_pages, v_pages, k_new, v_new, k_scale, v_scale, slot_mapping, page_size: int, err_flag=None,
                  stream=None) -> None:
    """Quantise k/v_new [B, H_kv, Dh] (bf16/fp16/fp32) to E4M3 with per-head fp32 scales [H_kv] and append them
    into uint8 pools [num_pages, H_kv, P, Dh]."""
    import torch

    num_pages, H_kv, P, Dh = k_pages.shape
    assert P == page_size and v_pages.shape == k_pages.shape and k_pages.dtype == torch.uint8
    B = k_new.shape[0]
    assert tuple(k_new.shape) == (B, H_kv, Dh) and v_new.shape == k_new.shape
    rc = lib().kv_append_fp8(_dev(k_pages, "k_pages"), _dev(v_pages, "v_pages", torch.uint8), _dev(k_new, "k_new"),
                             _dev(v_new, "v_new", k_new.dtype), _torch_dtype_code(k_new), _dev(k_scale, "k_scale", torch.float32),
                             _dev(v_scale, "v_scale", torch.float32), _dev(slot_mapping, "slot_mapping", torch.int64), B,
                             H_kv, Dh, page_size, num_pages, _dev(err_flag, "err_flag", torch.int32), _stream(stream))
    _check("kv_append_fp8", rc)


def paged_decode_attention_fp8(out, q, k_pages, v_pages, k_scale, v_scale, block_tables, seq_lens, scale: float,
                               num_splits: int = 0, workspace=None, err_flag=None, stream=None) -> None:
    """Decode over uint8 E4M3 pools [num_pages, H_kv, P, Dh] with per-head scales; q bf16/fp16 [B, H_q, Dh]."""
    import torch

    num_pages, H_kv, P, Dh = k_pages.shape
    B, H_q, Dh2 = q.shape
    assert Dh2 == Dh and v_pages.shape == k_pages.shape and k_pages.dtype == torch.uint8
    assert tuple(out.shape) == (B, H_q, Dh) and out.dtype == torch.float32
    max_blocks = block_tables.shape[1]
    rc = lib().paged_decode_attention_fp8(
        _dev(out, "out"), _dev(q, "q"), _torch_dtype_code(q), _dev(k_pages, "k_pages"), _dev(v_pages, "v_pages", torch.uint8),
        _dev(k_scale, "k_scale", torch.float32), _dev(v_scale, "v_scale", torch.float32),
        _dev(block_tables, "block_tables", torch.int32), max_blocks, _dev(seq_lens, "seq_lens", torch.int32), B, H_q,
        H_kv, Dh, P, num_pages, float(scale), num_splits, _dev(workspace, "workspace"),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _dev(err_flag, "err_flag", torch.int32),
        _stream(stream))
    _check("paged_decode_attention_fp8", rc)


def paged_decode_attention_rope_append(out, q, k_new, v_new, k_pages, v_pages, block_tables, seq_lens, cos_sin,
                                       scale: float, style: str = "half", num_splits: int = 0, workspace=None,
                                       err_flag=None, stream=None) -> None:
    """Rotate (q, the new k) at position seq_lens[b] - 1, append k / v, decode -- one launch (+ combine)."""
    import torch

    B, H_q, Dh = q.shape
    num_pages, H_kv, P, Dh2 = k_pages.shape
    assert Dh2 == Dh and v_pages.shape == k_pages.shape and tuple(out.shape) == (B, H_q, Dh)
    assert tuple(k_new.shape) == (B, H_kv, Dh) and v_new.shape == k_new.shape and cos_sin.shape[1] == Dh
    dt = k_pages.dtype
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().paged_decode_attention_rope_append(
        _dev(out, "out", torch.float32), _dev(q, "q", dt), _dev(k_new, "k_new", dt), _dev(v_new, "v_new", dt),
        _dev(k_pages, "k_pages"), _dev(v_pages, "v_pages", dt), _dev(block_tables, "block_tables", torch.int32),
        block_tables.shape[1], _dev(seq_lens, "seq_lens", torch.int32), _dev(cos_sin, "cos_sin", torch.float32),
        cos_sin.shape[0], ROPE_STYLE[style], B, H_q, H_kv, Dh, P, num_pages, float(scale), _torch_dtype_code(k_pages),
        num_splits, ws_ptr, ws_bytes, _dev(err_flag, "err_flag", torch.int32), _stream(stream))
    _check("paged_decode_attention_rope_append", rc)


def paged_prefill_attention(out, q, q_start, max_q_len: int, k_pages, v_pages, block_tables, seq_lens, scale: float,
                            err_flag=None, stream=None) -> None:
    """Causal attention of chunk rows q [N, H_q, Dh] (rows q_start[b] .. q_start[b+1]-1 are the last tokens of
    sequence b) over the paged cache; out fp32 [N, H_q, Dh]; q_start int32 [B + 1] (device)."""
    import torch

    num_pages, H_kv, P, Dh = k_pages.shape
    N, H_q, Dh2 = q.shape
    B = seq_lens.shape[0]
    assert Dh2 == Dh and v_pages.shape == k_pages.shape and tuple(out.shape) == (N, H_q, Dh)
    assert tuple(q_start.shape) == (B + 1,) and block_tables.shape[0] == B
    rc = lib().paged_prefill_attention(
        _dev(out, "out", torch.float32), _dev(q, "q", k_pages.dtype), _dev(q_start, "q_start", torch.int32),
        int(max_q_len), _dev(k_pages, "k_pages"), _dev(v_pages, "v_pages", k_pages.dtype),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1], _dev(seq_lens, "seq_lens", torch.int32),
        B, H_q, H_kv, Dh, P, num_pages, float(scale), _torch_dtype_code(k_pages), _dev(err_flag, "err_flag", torch.int32),
        _stream(stream))
    _check("paged_prefill_attention", rc)


KV_DECODE_KERNEL_AUTO, KV_DECODE_KERNEL_SIMT, KV_DECODE_KERNEL_MMA, KV_DECODE_KERNEL_TCGEN05 = 0, 1, 2, 3


def paged_decode_set_kernel(kind: int) -> None:
    _check("paged_decode_set_kernel", lib().paged_decode_set_kernel(kind))


def kv_copy_pages(k_pages, v_pages, src_pages, dst_pages, err_flag=None, stream=None) -> None:
    """Copy whole pages src_pages[i] -> dst_pages[i] of both pools (int32 device tensors)."""
    import torch

    num_pages, H_kv, P, Dh = k_pages.shape
    n = src_pages.numel()
    assert dst_pages.numel() == n and v_pages.shape == k_pages.shape
    rc = lib().kv_copy_pages(_dev(k_pages, "k_pages"), _dev(v_pages, "v_pages", k_pages.dtype),
                             _dev(src_pages, "src_pages", torch.int32) if n else None,
                             _dev(dst_pages, "dst_pages", torch.int32) if n else None, n, H_kv, Dh, P, num_pages,
                             _torch_dtype_code(k_pages), _dev(err_flag, "err_flag", torch.int32), _stream(stream))
    _check("kv_copy_pages", rc)


def paged_decode_num_splits(B: int, H_kv: int, max_blocks: int, page_size: int, num_splits: int = 0) -> int:
    out = ctypes.c_int32()
    _check("paged_decode_num_splits", lib().paged_decode_num_splits(B, H_kv, max_blocks, page_size, num_splits, out))
    return out.value


def paged_decode_launch_info(B: int, H_q: int, H_kv: int, Dh: int, max_blocks: int, page_size: int,
                             dtype: str = "bf16", num_splits: int = 0):
    """(split count, 0 = device-planned; kernel kind KV_DECODE_KERNEL_SIMT / _MMA / _TCGEN05)."""
    S, kind = ctypes.c_int32(), ctypes.c_int32()
    _check("paged_decode_launch_info", lib().paged_decode_launch_info(B, H_q, H_kv, Dh, max_blocks, page_size,
                                                                      DTYPE_CODE[dtype], num_splits, S, kind))
    return S.value, kind.value


def paged_decode_workspace_bytes(B: int, H_q: int, H_kv: int, Dh: int, max_blocks: int, page_size: int,
                                 num_splits: int = 0) -> int:
    out = ctypes.c_size_t()
    _check("paged_decode_workspace_bytes",
           lib().paged_decode_workspace_bytes(B, H_q, H_kv, Dh, max_blocks, page_size, num_splits, out))
    return out.value


def paged_decode_attention(out, q, k_pages, v_pages, block_tables, seq_lens, scale: float, num_splits: int = 0,
                           workspace=None, err_flag=None, stream=None) -> None:
    """out fp32 [B, H_q, Dh]; q [B, H_q, Dh]; k/v_pages [num_pages, H_kv, P, Dh];
    block_tables int32 [B, max_blocks]; seq_lens int32 [B] (all on the device)."""
    import torch

    B, H_q, Dh = q.shape
    num_pages, H_kv, P, Dh2 = k_pages.shape
    assert Dh2 == Dh and v_pages.shape == k_pages.shape and tuple(out.shape) == (B, H_q, Dh)
    assert block_tables.shape[0] == B and tuple(seq_lens.shape) == (B,)
    dt = _torch_dtype_code(k_pages)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().paged_decode_attention(
        _dev(out, "out", torch.float32), _dev(q, "q", k_pages.dtype), _dev(k_pages, "k_pages"),
        _dev(v_pages, "v_pages", k_pages.dtype), _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(seq_lens, "seq_lens", torch.int32), B, H_q, H_kv, Dh, P, num_pages, float(scale), dt, num_splits, ws_ptr,
        ws_bytes, _dev(err_flag, "err_flag", torch.int32), _stream(stream))
    _check("paged_decode_attention", rc)


def paged_decode_attention_append(out, q, k_new, v_new, k_pages, v_pages, block_tables, seq_lens, scale: float,
                                  num_splits: int = 0, workspace=None, err_flag=None, stream=None) -> None:
    """kv_append of the token at position seq_lens[b] - 1 and paged_decode_attention in one launch.
    k_new / v_new [B, H_kv, Dh] in the pools' dtype; other arguments as paged_decode_attention."""
    import torch

    B, H_q, Dh = q.shape
    num_pages, H_kv, P, Dh2 = k_pages.shape
    assert Dh2 == Dh and v_pages.shape == k_pages.shape and tuple(out.shape) == (B, H_q, Dh)
    assert tuple(k_new.shape) == (B, H_kv, Dh) and v_new.shape == k_new.shape
    assert block_tables.shape[0] == B and tuple(seq_lens.shape) == (B,)
    dt = _torch_dtype_code(k_pages)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr = _dev(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().paged_decode_attention_append(
        _dev(out, "out", torch.float32), _dev(q, "q", k_pages.dtype), _dev(k_new, "k_new", k_pages.dtype),
        _dev(v_new, "v_new", k_pages.dtype), _dev(k_pages, "k_pages"), _dev(v_pages, "v_pages", k_pages.dtype),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1], _dev(seq_lens, "seq_lens", torch.int32), B,
        H_q, H_kv, Dh, P, num_pages, float(scale), dt, num_splits, ws_ptr, ws_bytes, _dev(err_flag, "err_flag", torch.int32),
        _stream(stream))
    _check("paged_decode_attention_append", rc)


KV_NOALLOC_SCRATCH_BYTES = 8 * 1024 * 1024


def paged_decode_attention_noalloc(out, q, k_pages, v_pages, block_tables, seq_lens, scale: float, num_splits: int = 0,
                                   err_flag=None, stream=None) -> None:
    """paged_decode_attention for callers that cannot allocate device memory: the
    split partials live in the library's fixed device scratch (no workspace)."""
    import torch

    B, H_q, Dh = q.shape
    num_pages, H_kv, P, Dh2 = k_pages.shape
    assert Dh2 == Dh and v_pages.shape == k_pages.shape and tuple(out.shape) == (B, H_q, Dh)
    assert block_tables.shape[0] == B and tuple(seq_lens.shape) == (B,)
    dt = _torch_dtype_code(k_pages)
    rc = lib().paged_decode_attention_noalloc(
        _dev(out, "out", torch.float32), _dev(q, "q", k_pages.dtype), _dev(k_pages, "k_pages"),
        _dev(v_pages, "v_pages", k_pages.dtype), _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(seq_lens, "seq_lens", torch.int32), B, H_q, H_kv, Dh, P, num_pages, float(scale), dt, num_splits,
        _dev(err_flag, "err_flag", torch.int32), _stream(stream))
    _check("paged_decode_attention_noalloc", rc)


def exported_names() -> list:
    return [n for n, _, _ in SIGNATURES]
