"""FP8 (E4M3) K/V cache: quantising append and decode -- TEST INFRASTRUCTURE ONLY.

"03. KV Cache：用显存换计算" (the follow-up on KV quantisation) and the course
notes' table of KV-size levers (the row on storing each number in fewer bits: from 16 down to 8)
name storing K / V in 8 bits, with the warning that the error must be checked,
but fix no format. The plainest reading, taken here:

* Element format E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
  no infinities; S.1111.111 is NaN, so the largest finite value is 448;
  exponent field 0 holds subnormals m * 2^-9).
* One fp32 scale per KV head and pool (k_scale[h], v_scale[h]), chosen by the
  caller: stored code = E4M3(x / scale), read value = E4M3 value * scale.
* Quantising: x / scale in fp32 (IEEE division), then round to nearest even
  among the E4M3 values, saturating to +-448 (NaN stays NaN).
* Decode attention runs on the read values: score = scale_attn *
  sum_d q_d (k_d * k_scale), output = sum_t p_t (v_t * v_scale). q stays in
  its 16-bit storage type.

Exact arithmetic here (fp64); the codes are compared bit for bit.
"""
from __future__ import annotations

import numpy as np

from . import reference as R

E4M3_MAX = 448.0


def e4m3_value(code: int) -> float:
    """Value of one E4M3 code (NaN for S.1111.111), from the format definition."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
_POS = E4M3_TABLE[:0x7F]  # codes 0x00 .. 0x7E: 0 .. 448, increasing


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 codes -> fp64 values."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Round values to E4M3 codes: nearest, ties to the even code, saturating
    at 448; NaN -> 0x7F (with the sign bit of x)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # candidate codes below / above |x| among 0x00..0x7E
    hi = np.searchsorted(_POS, np.minimum(a, E4M3_MAX), side="left")
    hi = np.clip(hi, 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    d_lo = np.abs(a - _POS[lo])
    d_hi = np.abs(_POS[hi] - a)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(a >= E4M3_MAX, np.uint8(0x7E), code)
    sign = np.signbit(x).astype(np.uint8) << 7
    out = (code | sign).astype(np.uint8)
    out[np.isnan(x)] = (0x7F | sign[np.isnan(x)]).astype(np.uint8)
    return out


def quantize(raw: np.ndarray, dtype: str, scale_per_head: np.ndarray) -> np.ndarray:
    """Storage rows raw [N, H, Dh] of `dtype` -> E4M3 codes: E4M3(x / scale[h]),
    the division done in fp32."""
    x = R.decode_storage(raw, dtype).astype(np.float32)  # exact: 16-bit / fp32 values
    s = np.asarray(scale_per_head, dtype=np.float32)[None, :, None]
    return e4m3_encode((x / s).astype(np.float32))


def append_fp8(k_pool: np.ndarray, v_pool: np.ndarray, k_new, v_new, dtype: str, k_scale, v_scale, slots) -> None:
    """Quantise the new rows and write their codes at the slots (-1 skips)."""
    P = k_pool.shape[2]
    kq = quantize(k_new, dtype, k_scale)
    vq = quantize(v_new, dtype, v_scale)
    for b, slot in enumerate(np.asarray(slots, dtype=np.int64)):
        if slot < 0:
            continue
        k_pool[slot // P, :, slot % P, :] = kq[b]
        v_pool[slot // P, :, slot % P, :] = vq[b]


def paged_decode_fp8(q: np.ndarray, q_dtype: str, k_codes: np.ndarray, v_codes: np.ndarray, k_scale, v_scale,
                     block_tables: np.ndarray, seq_lens: np.ndarray, scale: float) -> np.ndarray:
    """fp64 decode over an E4M3 cache: per KV head h, the fp64 paged decode of
    the read values with the score scale folded as scale * k_scale[h] and the
    output multiplied by v_scale[h] (both exact rewritings of the definition)."""
    B, H_q, Dh = q.shape
    H_kv = k_codes.shape[1]
    g = H_q // H_kv
    qf = R.decode_storage(q, q_dtype).astype(np.float32)  # exact
    kf = e4m3_decode(k_codes).astype(np.float32)          # exact
    vf = e4m3_decode(v_codes).astype(np.float32)
    out = np.zeros((B, H_q, Dh), dtype=np.float64)
    ks = np.asarray(k_scale, dtype=np.float32).astype(np.float64)
    vs = np.asarray(v_scale, dtype=np.float32).astype(np.float64)
    for h in range(H_kv):
        pairs = [(b, hq) for b in range(B) for hq in range(h * g, (h + 1) * g)]
        part = R.paged_decode(qf, kf, vf, block_tables, seq_lens, float(scale) * ks[h], "fp32", pairs=pairs)
        out[:, h * g:(h + 1) * g, :] = part[:, h * g:(h + 1) * g, :] * vs[h]
    return out
