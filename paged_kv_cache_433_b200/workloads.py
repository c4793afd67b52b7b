"""Seeded synthetic inputs for paged decode attention.

This module only draws random numbers and describes workload shapes. It holds
none of the method's arithmetic (no paging, no slot math, no attention), so
both the CUDA path and the CPU oracle can take their inputs from it without
sharing any computation.

Every stream is a numpy ``Generator(PCG64)`` seeded from a ``SeedSequence`` of
``(config seed, stream kind, *indices)``, so one sequence's keys/values can be
regenerated on their own (used to check sampled outputs at full size).

Values are drawn N(0, 1) in float32 and rounded once to the storage dtype with
torch's round-to-nearest-even cast; the rounded bits are what both sides see.

Workload shapes follow the pages' examples:
  * tiny: lengths 35 and 12 at page size 16 ("06 KV Cache、Prefix Cache、
    PagedAttention 与 vLLM", section 6.5 block-16 / length-35 example).
  * Llama-3.1-8B-shaped decode layer: H_q=32, H_kv=8, Dh=128 ("03. KV Cache：
    用显存换计算" names Llama-3.1-8B; the GQA shape follows that model).
  * 32K long context, 32 layers, fp16: the KV-bytes worked example of
    "07｜KV Cache、FlashAttention与PagedAttention的内部过程", Q026 table.
  * shared-prefix batch and mixed continuous-batching sweep: section 6.4 and
    6.6 of the course-notes page.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np

# Stream kinds (second element of every SeedSequence entropy tuple).
S_LENGTHS = 1
S_PAGES = 2
S_Q = 3
S_K = 4
S_V = 5
S_KNEW = 6
S_VNEW = 7
S_TOKENS = 8
S_EVENTS = 9
S_SUFFIX = 10

DTYPES = ("fp32", "bf16", "fp16")
DTYPE_CODE = {"fp32": 0, "bf16": 1, "fp16": 2}
DTYPE_BYTES = {"fp32": 4, "bf16": 2, "fp16": 2}

VOCAB = 128256


def generator(seed: int, kind: int, *idx: int) -> np.random.Generator:
    """Independent PCG64 stream for (seed, kind, *idx)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(kind), *[int(i) for i in idx]])))


def round_to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values once to the storage dtype (RNE via torch casts).

    Returns the storage array: float32 for "fp32", uint16 bit patterns for
    "bf16"/"fp16".
    """
    import torch

    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "fp32":
        return x
    t = torch.from_numpy(x)
    if dtype == "bf16":
        return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    if dtype == "fp16":
        return t.to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    raise ValueError(f"unknown dtype {dtype}")


def normal_storage(seed: int, kind: int, idx: Sequence[int], shape: Tuple[int, ...], dtype: str) -> np.ndarray:
    """N(0,1) values of `shape`, rounded to `dtype` storage."""
    g = generator(seed, kind, *idx)
    x = g.standard_normal(size=shape, dtype=np.float32)
    return round_to_storage(x, dtype)


def page_order(num_pages: int, seed: int, idx: int = 0) -> np.ndarray:
    """Seeded random permutation of physical page ids 0..num_pages-1 (int32)."""
    g = generator(seed, S_PAGES, idx)
    return g.permutation(num_pages).astype(np.int32)


@dataclass(frozen=True)
class DecodeConfig:
    """Shape of one paged decode workload."""

    name: str
    dtype: str
    B: int
    H_q: int
    H_kv: int
    Dh: int
    page_size: int
    layers: int = 1
    seed: int = 0
    timed_steps: int = 100
    warmup_steps: int = 10

    @property
    def g(self) -> int:
        return self.H_q // self.H_kv

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.Dh))

    @property
    def elem_bytes(self) -> int:
        return DTYPE_BYTES[self.dtype]


# The five workloads. Names describe shape; lengths come from the functions below.
TINY = DecodeConfig("tiny-fp32-B2-len35+12-Hq4-Hkv2-Dh64-P16", "fp32", B=2, H_q=4, H_kv=2, Dh=64, page_size=16, seed=1)
LLAMA8B = DecodeConfig("llama3.1-8b-layer-bf16-B64-len512..4096-P16", "bf16", B=64, H_q=32, H_kv=8, Dh=128, page_size=16, seed=2)
LONG32K = DecodeConfig("long-context-fp16-B1-T32768-32layers-P16", "fp16", B=1, H_q=32, H_kv=8, Dh=128, page_size=16, layers=32, seed=3,
                       timed_steps=20, warmup_steps=3)
SHARED_PREFIX = DecodeConfig("shared-prefix-bf16-B32-prefix4096-suffix64..512-P16", "bf16", B=32, H_q=32, H_kv=8, Dh=128, page_size=16, seed=4)
TINY_POOL_PAGES = 8
LONG_T = 32768
PREFIX_LEN = 4096


def mixed_config(H_kv: int, page_size: int) -> DecodeConfig:
    return DecodeConfig(f"mixed-bf16-B256-lognormal1024-Hkv{H_kv}-P{page_size}", "bf16", B=256, H_q=32, H_kv=H_kv, Dh=128,
                        page_size=page_size, seed=5)


MIXED_POINTS = [(h, p) for h in (1, 8, 32) for p in (16, 32)]


def cached_lengths(cfg: DecodeConfig) -> np.ndarray:
    """Cached (pre-append) lengths per sequence, int64."""
    if cfg.seed == 1:
        return np.array([35, 12], dtype=np.int64)
    if cfg.seed == 2:
        g = generator(cfg.seed, S_LENGTHS)
        return g.integers(512, 4096, size=cfg.B, endpoint=True).astype(np.int64)
    if cfg.seed == 3:
        return np.full(cfg.B, LONG_T, dtype=np.int64)
    if cfg.seed == 4:
        g = generator(cfg.seed, S_LENGTHS)
        return PREFIX_LEN + g.integers(64, 512, size=cfg.B, endpoint=True).astype(np.int64)
    if cfg.seed == 5:
        return lognormal_lengths(cfg.B, generator(cfg.seed, S_LENGTHS, cfg.H_kv, cfg.page_size))
    raise ValueError(cfg.name)


def lognormal_lengths(n: int, g: np.random.Generator) -> np.ndarray:
    """Log-normal lengths: median 1024, sigma 1, clipped to [16, 16384]."""
    x = np.exp(np.log(1024.0) + g.standard_normal(n))
    return np.clip(np.rint(x), 16, 16384).astype(np.int64)


def ragged_lengths(B: int, page_size: int, seed: int, uniform: bool = False) -> np.ndarray:
    """Cached lengths for a many-row batch with the ragged cases a chunked
    launch meets: log-normal body (median 96 tokens, sigma 1), empty rows,
    rows that end exactly on a page boundary after the append, rows of 8, 16,
    65 and 130 whole pages after the append, and one long row (60 pages).
    uniform=True: every row 37 pages + 3 tokens after the append."""
    P = page_size
    if uniform:
        return np.full(B, 37 * P + 2, dtype=np.int64)
    g = generator(seed, S_LENGTHS, B, P)
    x = np.clip(np.rint(np.exp(np.log(96.0) + g.standard_normal(B))), 0, 40 * P).astype(np.int64)
    x[0::17] = 0
    x[1::23] = P - 1
    for i, pages in enumerate((8, 16, 65, 130)):
        x[5 + i::31] = pages * P - 1
    x[B // 2] = 60 * P - 7
    return x


@dataclass
class ChurnEvent:
    """One step of the mixed sweep: which batch slots exit and their new lengths."""

    exits: np.ndarray  # int64 indices of slots whose sequence finishes before this step
    new_lengths: np.ndarray  # cached length of the sequence admitted into each exiting slot


def churn_events(cfg: DecodeConfig, steps: int, exit_prob: float = 1.0 / 32.0) -> List[ChurnEvent]:
    """Per-step random exit/admit for the continuous-batching sweep."""
    g = generator(cfg.seed, S_EVENTS, cfg.H_kv, cfg.page_size)
    out = []
    for _ in range(steps):
        ex = np.nonzero(g.random(cfg.B) < exit_prob)[0].astype(np.int64)
        out.append(ChurnEvent(ex, lognormal_lengths(len(ex), g)))
    return out


@dataclass
class PrefixWorkload:
    """Token ids of the shared-prefix batch."""

    prefix: np.ndarray  # int32 [PREFIX_LEN]
    suffixes: List[np.ndarray]  # int32 per sequence
    divergence: np.ndarray  # int64 per sequence: index of the token changed in the probe prompt

    def tokens(self, b: int) -> np.ndarray:
        return np.concatenate([self.prefix, self.suffixes[b]]).astype(np.int32)

    def probe(self, b: int) -> np.ndarray:
        """Sequence b's prompt with the token at divergence[b] replaced by a different id."""
        t = self.tokens(b).copy()
        d = int(self.divergence[b])
        t[d] = (int(t[d]) + 1 + int(self.divergence[b] % 7)) % VOCAB
        return t


def prefix_workload(cfg: DecodeConfig = SHARED_PREFIX) -> PrefixWorkload:
    lens = cached_lengths(cfg)
    g = generator(cfg.seed, S_TOKENS)
    prefix = g.integers(0, VOCAB, size=PREFIX_LEN).astype(np.int32)
    suffixes = []
    for b in range(cfg.B):
        gs = generator(cfg.seed, S_SUFFIX, b)
        suffixes.append(gs.integers(0, VOCAB, size=int(lens[b]) - PREFIX_LEN).astype(np.int32))
    div = generator(cfg.seed, S_EVENTS).integers(0, lens, size=cfg.B).astype(np.int64)
    return PrefixWorkload(prefix, suffixes, div)


def kv_rows(cfg: DecodeConfig, layer: int, b: int, n: int, start: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Logical K and V rows [n, H_kv, Dh] of sequence b at `layer`, storage dtype.

    Rows are drawn per (layer, sequence) so a sample can be regenerated alone.
    `start` skips rows (they are drawn and dropped, so values do not depend on n).
    """
    shape = (start + n, cfg.H_kv, cfg.Dh)
    k = normal_storage(cfg.seed, S_K, (layer, b), shape, cfg.dtype)[start:]
    v = normal_storage(cfg.seed, S_V, (layer, b), shape, cfg.dtype)[start:]
    return k, v


def new_token_kv(cfg: DecodeConfig, layer: int, step: int) -> Tuple[np.ndarray, np.ndarray]:
    """K and V of the token appended at `step` for every sequence: [B, H_kv, Dh]."""
    shape = (cfg.B, cfg.H_kv, cfg.Dh)
    return (normal_storage(cfg.seed, S_KNEW, (layer, step), shape, cfg.dtype),
            normal_storage(cfg.seed, S_VNEW, (layer, step), shape, cfg.dtype))


def queries(cfg: DecodeConfig, layer: int, step: int) -> np.ndarray:
    """Decode queries [B, H_q, Dh] for `step`, storage dtype."""
    return normal_storage(cfg.seed, S_Q, (layer, step), (cfg.B, cfg.H_q, cfg.Dh), cfg.dtype)


def all_queries(cfg: DecodeConfig, layer: int, b: int, n: int) -> np.ndarray:
    """One query per position [n, H_q, Dh] (for full causal recompute on tiny inputs)."""
    return normal_storage(cfg.seed, S_Q, (layer, 1000 + b), (n, cfg.H_q, cfg.Dh), cfg.dtype)
