"""Oracle definitions (fp64) -- TEST INFRASTRUCTURE ONLY.

Each function restates one passage of the pages; see the package docstring
for the page titles behind the [KV-04] / [HB-07] / [CN-06] / [KV-03] tags.
Nothing here is blocked, fused or reordered beyond what the cited definition
states, so it can be checked against the pages by eye.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

from . import build_oracle

DT_CODE = {"fp32": 0, "bf16": 1, "fp16": 2}

# --------------------------------------------------------------------------
# Softmax and the online (m, l, u) merge -- [HB-07] Q027
# --------------------------------------------------------------------------


def softmax_weighted_sum(scores: Sequence[float], values: np.ndarray) -> np.ndarray:
    """o = sum_j softmax(s)_j v_j, the full (non-blocked) definition.

    [HB-07] Q027: the online merge must give the same result as a full softmax
    over all scores followed by the weighted sum.
    """
    s = np.asarray(scores, dtype=np.float64)
    v = np.asarray(values, dtype=np.float64)
    if v.ndim == 1:
        v = v[:, None]
    m = s.max()
    w = np.exp(s - m)
    return (w[:, None] * v).sum(axis=0) / w.sum()


def block_state(scores: Sequence[float], values: np.ndarray) -> Tuple[float, float, np.ndarray]:
    """State of one block: m = max s_j, l = sum exp(s_j - m), u = sum exp(s_j - m) v_j.

    [HB-07] Q027, "推导在线softmax合并" (the three maintained quantities).
    """
    s = np.asarray(scores, dtype=np.float64)
    v = np.asarray(values, dtype=np.float64)
    if v.ndim == 1:
        v = v[:, None]
    m = float(s.max())
    e = np.exp(s - m)
    return m, float(e.sum()), (e[:, None] * v).sum(axis=0)


def merge_block(state: Optional[Tuple[float, float, np.ndarray]], scores: Sequence[float], values: np.ndarray,
                rescale_old: bool = True) -> Tuple[float, float, np.ndarray]:
    """Fold one new block into the running (m_old, l_old, u_old).

    [HB-07] Q027: m_new = max(m_old, m_b); alpha = exp(m_old - m_new);
    l_new = alpha l_old + sum_new exp(s_j - m_new);
    u_new = alpha u_old + sum_new exp(s_j - m_new) v_j.
    `rescale_old=False` is the page's own counter-example (step 6 of its
    two-block table: the maximum is updated but the old sums are not scaled).
    """
    s = np.asarray(scores, dtype=np.float64)
    v = np.asarray(values, dtype=np.float64)
    if v.ndim == 1:
        v = v[:, None]
    if state is None:
        return block_state(s, v)
    m_old, l_old, u_old = state
    m_b = float(s.max())
    m_new = max(m_old, m_b)
    alpha = math.exp(m_old - m_new) if rescale_old else 1.0
    e = np.exp(s - m_new)
    return m_new, alpha * l_old + float(e.sum()), alpha * u_old + (e[:, None] * v).sum(axis=0)


def online_softmax(blocks: Iterable[Tuple[Sequence[float], np.ndarray]], rescale_old: bool = True):
    """Walk the blocks in order with the online merge; returns (m, l, u, o = u / l)."""
    st = None
    for s, v in blocks:
        st = merge_block(st, s, v, rescale_old=rescale_old)
    m, l, u = st
    return m, l, u, u / l


def merge_states(a: Tuple[float, float, np.ndarray], b: Tuple[float, float, np.ndarray]):
    """Merge two block states (the same rule with block b already summarised).

    This is how split partial results are combined: m* = max(m_a, m_b),
    l = e^{m_a-m*} l_a + e^{m_b-m*} l_b, u likewise ([HB-07] Q027).
    """
    ma, la, ua = a
    mb, lb, ub = b
    m = max(ma, mb)
    wa, wb = math.exp(ma - m), math.exp(mb - m)
    return m, wa * la + wb * lb, wa * ua + wb * ub


# --------------------------------------------------------------------------
# Full causal attention -- [KV-04] formula section; [KV-03] "注意力的公式"
# --------------------------------------------------------------------------


def causal_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(Q K^T * scale + causal_mask) V for every position of one sequence.

    Q [T, H_q, Dh], K/V [T, H_kv, Dh] (fp64). Query head h uses KV head
    h // (H_q // H_kv) (contiguous GQA grouping, the reading taken for
    [CN-06] 6.3). Returns O [T, H_q, Dh].
    """
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    T, H_q, Dh = Q.shape
    H_kv = K.shape[1]
    g = H_q // H_kv
    O = np.zeros((T, H_q, Dh))
    mask = np.triu(np.full((T, T), -np.inf), k=1)  # position i sees j <= i
    for h in range(H_q):
        kv = h // g
        S = Q[:, h, :] @ K[:, kv, :].T * scale + mask
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P /= P.sum(axis=1, keepdims=True)
        O[:, h, :] = P @ V[:, kv, :]
    return O


def decode_logical(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """One decode query per head against a logical (unpaged) history.

    q [H_q, Dh], K/V [T, H_kv, Dh]; the last query attends to all T positions
    ([HB-07] Q025: q_new @ K_all^T, softmax, weighted sum). Returns [H_q, Dh].
    """
    q = np.asarray(q, np.float64)
    H_q = q.shape[0]
    g = H_q // K.shape[1]
    out = np.zeros_like(q)
    if K.shape[0] == 0:
        return out
    for h in range(H_q):
        s = (np.asarray(K[:, h // g, :], np.float64) @ q[h]) * scale
        out[h] = softmax_weighted_sum(s, V[:, h // g, :])
    return out


# --------------------------------------------------------------------------
# Paging arithmetic -- [HB-07] Q028 block-size-4 example; [CN-06] 6.5
# --------------------------------------------------------------------------


def logical_block(pos: int, page_size: int) -> Tuple[int, int]:
    """(logical block, offset) of a position: pos // P and pos % P ([HB-07] Q028 steps 1-2)."""
    return pos // page_size, pos % page_size


def physical_slot(table_row: Sequence[int], page_size: int, pos: int) -> int:
    """Flat slot page * P + offset of position `pos` through a block-table row ([HB-07] Q028 step 3)."""
    blk, off = logical_block(pos, page_size)
    return int(table_row[blk]) * page_size + off


def needs_new_page(cached_len: int, page_size: int) -> bool:
    """Appending at position `cached_len` needs a fresh block exactly when the last one is full.

    [HB-07] Q028: with P=4 and 10 cached tokens, positions 10 and 11 fill the
    third block; position 12 is the first that needs a new block.
    """
    return cached_len % page_size == 0


def blocks_for_len(length: int, page_size: int) -> Tuple[int, int, int]:
    """(blocks, slots, wasted) for a sequence of `length` tokens ([CN-06] 6.5: 35 @ 16 -> 3, 48, 13)."""
    blocks = -(-length // page_size)
    slots = blocks * page_size
    return blocks, slots, slots - length


def kv_cache_bytes(L: int, B: int, T: int, H_kv: int, Dh: int, bytes_per_elem: int) -> int:
    """KV bytes = 2 * L * B * T * H_kv * Dh * bytes ([HB-07] Q026; [CN-06] 6.3)."""
    return 2 * L * B * T * H_kv * Dh * bytes_per_elem


def kv_cache_bytes_ragged(L: int, lengths: Sequence[int], H_kv: int, Dh: int, bytes_per_elem: int) -> int:
    """Same, with sum_i T_i in place of B * T for unequal lengths ([CN-06] 6.3)."""
    return 2 * L * int(sum(int(t) for t in lengths)) * H_kv * Dh * bytes_per_elem


def scatter_to_pages(pool: np.ndarray, table_row: Sequence[int], rows: np.ndarray, start: int = 0) -> None:
    """Write logical rows [n, H_kv, Dh] at positions start.. into pool [pages, H_kv, P, Dh] (in place).

    Position t goes to page table_row[t // P], offset t % P (vectorised over t).
    """
    P = pool.shape[2]
    t = np.arange(start, start + rows.shape[0])
    pages = np.asarray(table_row, dtype=np.int64)[t // P]
    pool[pages, :, t % P, :] = rows


# --------------------------------------------------------------------------
# fp64 paged decode in C (OpenMP over (sequence, query head))
# --------------------------------------------------------------------------

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = build_oracle.build()
        lib = ctypes.CDLL(path)
        lib.oracle_paged_decode.restype = ctypes.c_int
        lib.oracle_paged_decode.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
            ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
            ctypes.c_double, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32]
        lib.oracle_decode_storage.restype = None
        lib.oracle_decode_storage.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32]
        lib.oracle_max_threads.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def max_threads() -> int:
    return int(_lib().oracle_max_threads())


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def decode_storage(raw: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array (float32 or uint16 bits) -> fp64 numbers, same shape."""
    raw = np.ascontiguousarray(raw)
    out = np.empty(raw.shape, dtype=np.float64)
    _lib().oracle_decode_storage(_ptr(out), _ptr(raw), raw.size, DT_CODE[dtype])
    return out


def paged_decode(q: np.ndarray, k_pages: np.ndarray, v_pages: np.ndarray, block_tables: np.ndarray,
                 seq_lens: np.ndarray, scale: float, dtype: str,
                 pairs: Optional[Sequence[Tuple[int, int]]] = None, nthreads: int = 0) -> np.ndarray:
    """fp64 decode attention over a paged cache (full score row + full softmax).

    q [B, H_q, Dh], k/v_pages [num_pages, H_kv, P, Dh] (storage dtype),
    block_tables int32 [B, max_blocks], seq_lens int32 [B] (including the
    token appended this step). Returns fp64 [B, H_q, Dh]; with `pairs`, only
    those (b, h) rows are computed (the rest are zero).
    """
    q = np.ascontiguousarray(q)
    k_pages = np.ascontiguousarray(k_pages)
    v_pages = np.ascontiguousarray(v_pages)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, H_q, Dh = q.shape
    num_pages, H_kv, P, Dh2 = k_pages.shape
    assert Dh2 == Dh and v_pages.shape == k_pages.shape and bt.shape[0] == B and sl.shape == (B,)
    out = np.zeros((B, H_q, Dh), dtype=np.float64)
    pr = None
    n_pairs = 0
    if pairs is not None:
        pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        n_pairs = pr.shape[0]
    rc = _lib().oracle_paged_decode(_ptr(out), _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(bt), bt.shape[1], _ptr(sl),
                                    B, H_q, H_kv, Dh, P, num_pages, float(scale), DT_CODE[dtype],
                                    _ptr(pr) if pr is not None else None, n_pairs, int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_paged_decode failed: {rc}")
    return out


# --------------------------------------------------------------------------
# Multi-token query over the paged cache (chunked prefill / prompt extension)
# --------------------------------------------------------------------------


def chunk_positions(q_start: Sequence[int], seq_lens: Sequence[int]) -> np.ndarray:
    """Position of every query row: the chunk of sequence b is its last
    n_b = q_start[b+1] - q_start[b] tokens, at positions seq_lens[b] - n_b ...
    seq_lens[b] - 1 ([CN-06] 6.2: a prefill chunk is processed after the part
    of the prompt already cached; 6.6 chunked prefill)."""
    qs = np.asarray(q_start, dtype=np.int64)
    sl = np.asarray(seq_lens, dtype=np.int64)
    pos = np.empty(int(qs[-1]), dtype=np.int64)
    for b in range(len(sl)):
        n = int(qs[b + 1] - qs[b])
        pos[qs[b]:qs[b + 1]] = sl[b] - n + np.arange(n)
    return pos


def paged_prefill(q: np.ndarray, q_start: Sequence[int], k_pages: np.ndarray, v_pages: np.ndarray,
                  block_tables: np.ndarray, seq_lens: Sequence[int], scale: float, dtype: str) -> np.ndarray:
    """fp64 causal attention of a chunk of query rows over the paged cache.

    q [N, H_q, Dh] (N = q_start[-1] rows; rows q_start[b] .. q_start[b+1]-1
    belong to sequence b). The query at position p attends to the keys at
    positions 0 .. p (the causal rule of [KV-04] / [HB-07] Q025: a token sees
    itself and everything before it), i.e. it is exactly a decode over a
    sequence of length p + 1 that shares sequence b's block table. Each row is
    computed that way by the fp64 decode above.
    """
    qs = np.asarray(q_start, dtype=np.int64)
    B = len(seq_lens)
    pos = chunk_positions(qs, seq_lens)
    owner = np.repeat(np.arange(B), np.diff(qs))
    tables = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32)[owner])
    lens = (pos + 1).astype(np.int32)
    return paged_decode(q, k_pages, v_pages, tables, lens, scale, dtype)
