"""Rotary position embedding of q / k before the KV append -- TEST INFRASTRUCTURE ONLY.

[CN-06] 6.1 gives the per-layer order for a new token: project q, k, v; rotate
q and k by the token's position; append k and v to the cache; then attend.
The pages name the rotation but do not define it, so the plainest reading is
taken (the rotary embedding as usually defined):

* Dimension pairs (i, j) are rotated by the angle pos * theta_k, with
  theta_k = base ** (-2k / Dh) for pair k = 0 .. Dh/2 - 1:
      x_i' = x_i cos - x_j sin,     x_j' = x_j cos + x_i sin.
* Two pairings are in use and both are provided: "half" pairs dimension k
  with k + Dh/2 (the split-halves layout of Llama-family checkpoints), and
  "interleaved" pairs 2k with 2k + 1 (the original formulation).
* The cos / sin values come from a table [max_pos][Dh] of fp32 numbers
  (cos in columns 0 .. Dh/2 - 1, sin in Dh/2 .. Dh - 1), computed here in
  fp64 and rounded once to fp32; the caller of the CUDA path passes the same
  table in.
* Stored precision: the rotation of stored values is done in fp32 with each
  product and the sum rounded separately (no fused multiply-add), then the
  result is rounded to the storage dtype with round-to-nearest-even. This
  fixes every rounding, so the stored bits are reproducible exactly.

`rotate_fp64` is the exact rotation (the definition); `apply_rope` is the
stored-precision version the CUDA path must match bit for bit.
"""
from __future__ import annotations

import numpy as np

STYLES = ("half", "interleaved")
STYLE_CODE = {"half": 0, "interleaved": 1}


def pair_index(Dh: int, style: str):
    """Index arrays (i, j) of the rotated pairs, pair k first."""
    if Dh % 2:
        raise ValueError("Dh must be even")
    k = np.arange(Dh // 2)
    if style == "half":
        return k, k + Dh // 2
    if style == "interleaved":
        return 2 * k, 2 * k + 1
    raise ValueError(style)


def angles(positions, Dh: int, base: float) -> np.ndarray:
    """fp64 angles pos * theta_k, shape [len(positions), Dh/2]."""
    pos = np.asarray(positions, dtype=np.float64).reshape(-1, 1)
    k = np.arange(Dh // 2, dtype=np.float64)
    theta = np.power(float(base), -2.0 * k / Dh)
    return pos * theta[None, :]


def rope_table(max_pos: int, Dh: int, base: float = 10000.0) -> np.ndarray:
    """fp32 table [max_pos][Dh]: cos(pos theta_k) in column k, sin in column Dh/2 + k."""
    a = angles(np.arange(max_pos), Dh, base)
    return np.concatenate([np.cos(a), np.sin(a)], axis=1).astype(np.float32)


def rotate_fp64(x: np.ndarray, positions, Dh: int, base: float, style: str) -> np.ndarray:
    """Exact rotation of fp64 rows x [N, ..., Dh] by their positions [N]."""
    x = np.asarray(x, dtype=np.float64)
    a = angles(positions, Dh, base)  # [N, Dh/2]
    shape = (x.shape[0],) + (1,) * (x.ndim - 2) + (Dh // 2,)
    c = np.cos(a).reshape(shape)
    s = np.sin(a).reshape(shape)
    i, j = pair_index(Dh, style)
    out = x.copy()
    out[..., i] = x[..., i] * c - x[..., j] * s
    out[..., j] = x[..., j] * c + x[..., i] * s
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 with round-to-nearest-even; uint16 bit patterns.
    NaN stays NaN (quiet)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    rounded[nan] = ((b[nan] >> 16) | 0x40).astype(np.uint16)
    return rounded


def to_storage(x32: np.ndarray, dtype: str) -> np.ndarray:
    """fp32 values -> storage array (float32, or uint16 bits for bf16 / fp16), RNE."""
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    if dtype == "fp32":
        return x32
    if dtype == "bf16":
        return f32_to_bf16_bits(x32)
    if dtype == "fp16":
        return x32.astype(np.float16).view(np.uint16)
    raise ValueError(dtype)


def storage_to_f32(raw: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array -> fp32 values (exact)."""
    raw = np.ascontiguousarray(raw)
    if dtype == "fp32":
        return raw.astype(np.float32)
    if dtype == "bf16":
        return (raw.astype(np.uint32) << 16).view(np.float32)
    if dtype == "fp16":
        return raw.view(np.float16).astype(np.float32)
    raise ValueError(dtype)


def apply_rope(raw: np.ndarray, positions, table: np.ndarray, style: str, dtype: str) -> np.ndarray:
    """Stored-precision rotation of storage rows raw [N, H, Dh] by positions [N].

    Per pair, in fp32: p1 = x_i * c, p2 = x_j * s, x_i' = p1 - p2;
    p3 = x_j * c, p4 = x_i * s, x_j' = p3 + p4; each operation rounded to
    fp32, then x' rounded to the storage dtype.
    """
    N, H, Dh = raw.shape
    x = storage_to_f32(raw, dtype)
    pos = np.asarray(positions, dtype=np.int64)
    c = table[pos, : Dh // 2][:, None, :].astype(np.float32)
    s = table[pos, Dh // 2:][:, None, :].astype(np.float32)
    i, j = pair_index(Dh, style)
    xi, xj = x[..., i], x[..., j]
    out = x.copy()
    out[..., i] = (xi * c).astype(np.float32) - (xj * s).astype(np.float32)
    out[..., j] = (xj * c).astype(np.float32) + (xi * s).astype(np.float32)
    return to_storage(out.astype(np.float32), dtype)


def rope_append(k_pool: np.ndarray, v_pool: np.ndarray, k_new: np.ndarray, v_new: np.ndarray, slots, positions,
                table: np.ndarray, style: str, dtype: str) -> None:
    """[CN-06] 6.1 order: rotate the new k by its position, then write k and v
    into their slots (pool[slot // P, :, slot % P, :]); slot -1 skips the row."""
    P = k_pool.shape[2]
    k_rot = apply_rope(k_new, positions, table, style, dtype)
    for b, slot in enumerate(np.asarray(slots, dtype=np.int64)):
        if slot < 0:
            continue
        k_pool[slot // P, :, slot % P, :] = k_rot[b]
        v_pool[slot // P, :, slot % P, :] = v_new[b]
