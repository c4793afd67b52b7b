"""Build one paged decode step twice: through the product (C ABI + CUDA) and
through the oracle, from the same seeded inputs, sharing no computation.

Product side: KvPool allocates pages, kv_slots_for_range + kv_append write the
cached K/V (a prefill-style append), kv_append_slots + kv_append add the new
token, paged_decode_attention attends.
Oracle side: PoolModel allocates, scatter_to_pages writes, append_slots adds
the new token, reference.paged_decode attends in fp64.
Block tables, slots and the physical pools are compared bit-exactly; the
attention output within the dtype's tolerance.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np
import torch

from helpers import TOL
from oracle import reference as R
from oracle.pool_model import PoolModel
from paged_kv_cache_433_b200 import kvpaged as K
from paged_kv_cache_433_b200 import workloads as W

TORCH_DT = {"fp32": torch.float32, "bf16": torch.bfloat16, "fp16": torch.float16}
NAN_BITS = {"bf16": np.uint16(0x7FC0), "fp16": np.uint16(0x7E00)}


def to_device(raw: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(raw))
    if dtype != "fp32":
        t = t.view(torch.int16).view(TORCH_DT[dtype])
    return t.cuda()


def device_bits(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.float32:
        return t.cpu().view(torch.int32).numpy().view(np.uint32)
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def oracle_pool(num_pages, cfg):
    shape = (num_pages, cfg.H_kv, cfg.page_size, cfg.Dh)
    if cfg.dtype == "fp32":
        return np.full(shape, np.nan, np.float32), np.full(shape, np.nan, np.float32)
    return np.full(shape, NAN_BITS[cfg.dtype], np.uint16), np.full(shape, NAN_BITS[cfg.dtype], np.uint16)


def check_close(gpu: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    atol, rtol = TOL[dtype]
    err = np.abs(gpu.astype(np.float64) - ref)
    bad = err > atol + rtol * np.abs(ref)
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    assert not bad.any(), f"{what}: {bad.sum()} / {bad.size} outside tol; max err {err.max():.3e}"
    return float(err.max())


@dataclass
class Step:
    """Everything one decode step needs on both sides."""

    cfg: W.DecodeConfig
    lens: np.ndarray                 # cached lengths before the append
    num_pages: int
    max_blocks: int
    # product
    pool: K.KvPool = None
    tab: np.ndarray = None           # int32 [B, max_blocks]
    k_pages: torch.Tensor = None
    v_pages: torch.Tensor = None
    # oracle
    mpool: PoolModel = None
    mtab: List[List[int]] = None
    kp: np.ndarray = None
    vp: np.ndarray = None
    logical_k: list = field(default_factory=list)
    logical_v: list = field(default_factory=list)


def build_cache(cfg: W.DecodeConfig, lens: Sequence[int], layer: int = 0, slack_pages: int = 4,
                extra_blocks: int = 1, keep_logical: bool = False, max_blocks: Optional[int] = None) -> Step:
    """Allocate and fill the cache of `lens` tokens per sequence on both sides."""
    lens = np.asarray(lens, dtype=np.int64)
    P = cfg.page_size
    B = len(lens)
    need = [-(-(int(L) + 1) // P) for L in lens]
    if max_blocks is None:
        max_blocks = max(need) + extra_blocks
    num_pages = int(sum(need)) + slack_pages
    order = W.page_order(num_pages, cfg.seed, layer)
    st = Step(cfg, lens, num_pages, max_blocks)
    st.pool = K.KvPool(num_pages, P, order)
    st.mpool = PoolModel(num_pages, P, order)
    st.tab = np.full((B, max_blocks), -1, np.int32)
    st.mtab = [[-1] * max_blocks for _ in range(B)]
    for b in range(B):
        k = -(-int(lens[b]) // P)
        ids = st.pool.alloc(k)
        st.tab[b, :k] = ids
        st.mtab[b][:k] = st.mpool.alloc(k)
    assert st.tab.tolist() == st.mtab, "block tables differ from the pool model"

    dt = TORCH_DT[cfg.dtype]
    shape = (num_pages, cfg.H_kv, P, cfg.Dh)
    st.k_pages = torch.full(shape, float("nan"), dtype=dt, device="cuda")
    st.v_pages = torch.full(shape, float("nan"), dtype=dt, device="cuda")
    st.kp, st.vp = oracle_pool(num_pages, cfg)
    # product: prefill-style kv_append calls over chunks of sequences
    slots_all, ks, vs = [], [], []
    for b in range(B):
        L = int(lens[b])
        if L > 0:
            slots = K.kv_slots_for_range(st.tab[b], P, 0, L)
            kr, vr = W.kv_rows(cfg, layer, b, L)
            R.scatter_to_pages(st.kp, st.mtab[b], kr)
            R.scatter_to_pages(st.vp, st.mtab[b], vr)
            if keep_logical:
                st.logical_k.append(kr)
                st.logical_v.append(vr)
            slots_all.append(slots)
            ks.append(to_device(kr, cfg.dtype))
            vs.append(to_device(vr, cfg.dtype))
        if sum(len(s) for s in slots_all) > (1 << 22) or b == B - 1:
            if slots_all:
                sl = torch.from_numpy(np.concatenate(slots_all)).cuda()
                K.kv_append(st.k_pages, st.v_pages, torch.cat(ks), torch.cat(vs), sl, P)
                slots_all, ks, vs = [], [], []
    torch.cuda.synchronize()
    return st


def append_and_decode(st: Step, layer: int = 0, step: int = 0, num_splits: int = 0, check_pools: bool = True,
                      sample: Optional[Sequence[int]] = None, fused: bool = False):
    """New token append + decode on both sides. Returns (gpu_out fp32 np, ref fp64 np, err_flag).

    fused=True appends through paged_decode_attention_append (one launch) instead of
    kv_append followed by paged_decode_attention."""
    cfg = st.cfg
    P = cfg.page_size
    B = len(st.lens)
    lens32 = st.lens.astype(np.int32).copy()
    mlens = [int(x) for x in st.lens]
    slots = st.pool.append_slots(st.tab, lens32)
    mslots = st.mpool.append_slots(st.mtab, st.max_blocks, mlens)
    assert list(slots) == mslots and st.tab.tolist() == st.mtab and lens32.tolist() == mlens

    k_new, v_new = W.new_token_kv(cfg, layer, step)
    q = W.queries(cfg, layer, step)
    k_new, v_new, q = k_new[:B], v_new[:B], q[:B]  # a test may run the first B rows of a config
    # oracle side: write the new token at its slot, then fp64 decode
    for b in range(B):
        page, off = divmod(mslots[b], P)
        st.kp[page, :, off, :] = k_new[b]
        st.vp[page, :, off, :] = v_new[b]
    pairs = None
    if sample is not None:
        pairs = [(b, h) for b in sample for h in range(cfg.H_q)]
    ref = R.paged_decode(q, st.kp, st.vp, np.asarray(st.mtab, np.int32), np.asarray(mlens, np.int32), cfg.scale,
                         cfg.dtype, pairs=pairs)

    # product side
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty((B, cfg.H_q, cfg.Dh), dtype=torch.float32, device="cuda")
    ws_bytes = K.paged_decode_workspace_bytes(B, cfg.H_q, cfg.H_kv, cfg.Dh, st.max_blocks, P, num_splits)
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    if fused:
        K.paged_decode_attention_append(out, to_device(q, cfg.dtype), to_device(k_new, cfg.dtype),
                                        to_device(v_new, cfg.dtype), st.k_pages, st.v_pages,
                                        torch.from_numpy(st.tab).cuda(), torch.from_numpy(lens32).cuda(), cfg.scale,
                                        num_splits=num_splits, workspace=ws, err_flag=err)
    else:
        K.kv_append(st.k_pages, st.v_pages, to_device(k_new, cfg.dtype), to_device(v_new, cfg.dtype),
                    torch.from_numpy(slots).cuda(), P, err_flag=err)
        K.paged_decode_attention(out, to_device(q, cfg.dtype), st.k_pages, st.v_pages, torch.from_numpy(st.tab).cuda(),
                                 torch.from_numpy(lens32).cuda(), cfg.scale, num_splits=num_splits, workspace=ws,
                                 err_flag=err)
    torch.cuda.synchronize()
    st.lens = st.lens + 1
    if check_pools:
        assert np.array_equal(device_bits(st.k_pages), st.kp.view(np.uint32) if cfg.dtype == "fp32" else st.kp), "K pool bits"
        assert np.array_equal(device_bits(st.v_pages), st.vp.view(np.uint32) if cfg.dtype == "fp32" else st.vp), "V pool bits"
    return out.cpu().numpy(), ref, int(err.item())


def replace_sequence(st: Step, b: int, new_len: int, tag: int) -> None:
    """Sequence in row b finishes (pages freed) and a new one of new_len cached tokens is admitted."""
    cfg = st.cfg
    P = cfg.page_size
    old = [p for p in st.mtab[b] if p >= 0]
    st.pool.free(old)
    st.mpool.free_pages(old)
    k = -(-new_len // P)
    st.tab[b, :] = -1
    st.tab[b, :k] = st.pool.alloc(k)
    st.mtab[b] = [-1] * st.max_blocks
    st.mtab[b][:k] = st.mpool.alloc(k)
    assert st.tab[b].tolist() == st.mtab[b]
    kr, vr = W.kv_rows(cfg, tag, b, new_len)
    R.scatter_to_pages(st.kp, st.mtab[b], kr)
    R.scatter_to_pages(st.vp, st.mtab[b], vr)
    sl = torch.from_numpy(K.kv_slots_for_range(st.tab[b], P, 0, new_len)).cuda()
    K.kv_append(st.k_pages, st.v_pages, to_device(kr, cfg.dtype), to_device(vr, cfg.dtype), sl, P)
    lens = st.lens.copy()
    lens[b] = new_len
    st.lens = lens
