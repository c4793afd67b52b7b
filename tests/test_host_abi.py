"""CPU tests of the C ABI: symbols, host pool / prefix index / slot bookkeeping
against the oracle's plain models, and argument checks (no GPU needed)."""
import os
import re
import subprocess

import numpy as np
import pytest

from helpers import ROOT, golden
from oracle.pool_model import PoolError, PoolModel, PrefixModel
from paged_kv_cache_433_b200 import kvpaged as K
from paged_kv_cache_433_b200 import workloads as W

HEADER = os.path.join(ROOT, "include", "kvpaged.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_433_b200 import build

    build.build()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    declared = header_functions()
    assert "paged_decode_attention" in declared and "kv_append" in declared and len(declared) >= 20
    out = subprocess.run(["nm", "-D", "--defined-only", K.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = [f for f in declared if f not in exported]
    assert not missing, missing
    assert sorted(K.exported_names()) == declared  # the binding covers the whole header
    L = K.lib()
    for f in declared:
        assert getattr(L, f) is not None


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(K, "_LIB", None)
    monkeypatch.setattr(K, "LIB_PATH", "/nonexistent/libkvpaged.so")
    with pytest.raises(RuntimeError):
        K.lib()


def test_product_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "paged_kv_cache_433_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".cpp", ".h")):
                src = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(from|import)\s+oracle", src, flags=re.M), f
                assert "decode_ref" not in src and "liboracle" not in src, f


# ------------------------------------------------------------------ pins
def test_blocks_and_bytes_pins():
    gd = golden("fragmentation.json")
    assert K.kv_blocks_for_len(gd["length"], gd["page_size"]) == (gd["blocks"], gd["slots"], gd["wasted"])
    for c in golden("kv_bytes.json")["cases"]:
        assert K.kv_cache_bytes(c["L"], c["B"], c["T"], c["H_kv"], c["Dh"], c["bytes"]) == c["total_bytes"]
    gd = golden("block_table_example.json")
    lk = gd["lookup"]
    assert K.kv_slot_for_pos(gd["table"], gd["page_size"], lk["pos"]) == lk["physical_page"] * gd["page_size"] + lk["offset"]
    slots = K.kv_slots_for_range(gd["table"], gd["page_size"], 10, 2)
    assert list(slots) == [a["page"] * gd["page_size"] + a["offset"] for a in gd["appends"]]
    with pytest.raises(K.KvError):
        K.kv_slot_for_pos(gd["table"], gd["page_size"], gd["first_position_needing_new_block"])


def test_append_slots_block_table_example():
    gd = golden("block_table_example.json")
    P = gd["page_size"]
    order = [7, 2, 19] + [i for i in range(24) if i not in (7, 2, 19)]
    pool = K.KvPool(24, P, order)
    tab = np.full((1, 5), -1, np.int32)
    tab[0, :3] = pool.alloc(3)
    lens = np.array([gd["cached_len"]], np.int32)
    assert list(pool.append_slots(tab, lens)) == [19 * P + 2]
    assert list(pool.append_slots(tab, lens)) == [19 * P + 3]
    nf = pool.num_free()
    assert list(pool.append_slots(tab, lens)) == [order[3] * P]
    assert pool.num_free() == nf - 1 and tab[0, 3] == order[3] and lens[0] == 13


# ------------------------------------------------------------------ pool vs model
def _kind(e: K.KvError) -> str:
    return e.name


@pytest.mark.parametrize("seed", range(6))
def test_pool_matches_model_random_ops(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(4, 40))
    order = rng.permutation(n).astype(np.int32)
    pool, model = K.KvPool(n, 16, order), PoolModel(n, 16, order)
    held = []
    for _ in range(300):
        op = rng.integers(0, 4)
        if op == 0:
            k = int(rng.integers(0, 6))
            exp_err = None
            try:
                want = model.alloc(k)
            except PoolError as e:
                exp_err = e.kind
            try:
                got = list(pool.alloc(k))
                assert exp_err is None and got == want
                held.extend(got)
            except K.KvError as e:
                assert _kind(e) == exp_err
        elif op == 1 and held:
            k = int(rng.integers(1, 4))
            ids = [held[int(i)] for i in rng.integers(0, len(held), k)]
            if rng.random() < 0.1:
                ids.append(int(rng.integers(-2, n + 2)))
            exp_err = None
            try:
                model.free_pages(ids)
            except PoolError as e:
                exp_err = e.kind
            try:
                pool.free(ids)
                assert exp_err is None
                for i in ids:
                    held.remove(i)
            except K.KvError as e:
                assert _kind(e) == exp_err
        elif op == 2 and held:
            ids = [held[int(i)] for i in rng.integers(0, len(held), 2)]
            if rng.random() < 0.2:
                ids.append(int(rng.integers(0, n)))
            exp_err = None
            try:
                model.incref(ids)
            except PoolError as e:
                exp_err = e.kind
            try:
                pool.incref(ids)
                assert exp_err is None
                held.extend(ids)
            except K.KvError as e:
                assert _kind(e) == exp_err
        assert pool.num_free() == model.num_free()
        for p in range(n):
            assert pool.refcount(p) == model.refcount(p)
    # the FIFO order of the free list is observable through alloc
    assert list(pool.alloc(pool.num_free())) == model.alloc(model.num_free())


@pytest.mark.parametrize("P", [4, 16, 32])
def test_append_slots_matches_model(P):
    rng = np.random.default_rng(P)
    B, max_blocks, n = 7, 12, 80
    order = rng.permutation(n).astype(np.int32)
    pool, model = K.KvPool(n, P, order), PoolModel(n, P, order)
    lens0 = rng.integers(0, 5 * P, B)
    tab = np.full((B, max_blocks), -1, np.int32)
    mtab = [[-1] * max_blocks for _ in range(B)]
    for b in range(B):
        k = -(-int(lens0[b]) // P)
        ids = pool.alloc(k)
        assert list(ids) == model.alloc(k)
        tab[b, :k] = ids
        mtab[b][:k] = list(ids)
    lens = lens0.astype(np.int32).copy()
    mlens = [int(x) for x in lens0]
    for step in range(3 * P):
        try:
            want = model.append_slots(mtab, max_blocks, mlens)
        except PoolError as e:
            with pytest.raises(K.KvError) as ei:
                pool.append_slots(tab, lens)
            assert ei.value.name == e.kind
            break
        got = pool.append_slots(tab, lens)
        assert list(got) == want and tab.tolist() == mtab and lens.tolist() == mlens


def test_append_slots_errors():
    pool = K.KvPool(8, 4)
    t = pool.alloc(1)
    pool.incref(t)
    tab = np.array([[t[0], -1], [t[0], -1]], np.int32)
    lens = np.array([2, 2], np.int32)
    with pytest.raises(K.KvError) as e:
        pool.append_slots(tab, lens)
    assert e.value.name == "SHARED_TAIL" and lens.tolist() == [2, 2]
    small = K.KvPool(1, 4)
    tab = np.full((2, 2), -1, np.int32)
    lens = np.zeros(2, np.int32)
    with pytest.raises(K.KvError) as e:
        small.append_slots(tab, lens)
    assert e.value.name == "OOM" and small.num_free() == 1 and lens.tolist() == [0, 0]
    full = np.array([[0]], np.int32)
    with pytest.raises(K.KvError) as e:
        small.append_slots(full, np.array([4], np.int32))
    assert e.value.name == "ARG"


def test_pool_argument_errors():
    with pytest.raises(K.KvError):
        K.KvPool(0, 16)
    with pytest.raises(K.KvError):
        K.KvPool(3, 16, [0, 0, 1])
    pool = K.KvPool(3, 16)
    with pytest.raises(K.KvError) as e:
        pool.refcount(3)
    assert e.value.name == "BAD_ID"


# ------------------------------------------------------------------ prefix index vs model
def test_prefix_demo_through_c_index():
    gd = golden("prefix_demo.json")
    P = gd["page_size_reading"]
    pool = K.KvPool(16, P)
    ix = K.KvPrefixIndex(P)
    cached = [ord(c) for c in gd["cached"]]
    pages = pool.alloc(3)
    ix.register(pool, cached, pages)
    hit = ix.match([ord(c) for c in gd["request"]])
    assert list(hit) == [pages[0]] and len(hit) * P == gd["reusable_tokens"]
    assert len(ix.match([ord(c) for c in gd["edit_at_start"]["request"]])) == 0


def test_shared_prefix_workload_divergence_points():
    """Shared-prefix batch: a probe that changes token d matches floor(d / 16) pages."""
    cfg = W.SHARED_PREFIX
    wl = W.prefix_workload(cfg)
    P = cfg.page_size
    lens = W.cached_lengths(cfg)
    n_pages = int(sum(-(-int(L) // P) for L in lens)) + 8
    pool = K.KvPool(n_pages, P, W.page_order(n_pages, cfg.seed))
    ix = K.KvPrefixIndex(P, salt=0x5EED)
    prefix_pages = pool.alloc(W.PREFIX_LEN // P)
    ix.register(pool, wl.prefix, prefix_pages)
    for b in range(cfg.B):
        toks = wl.tokens(b)
        hit = ix.match(toks)
        assert list(hit) == list(prefix_pages)
        pool.incref(hit)
        own = pool.alloc(-(-len(toks) // P) - len(hit))
        ix.register(pool, toks, np.concatenate([hit, own]))
    for b in range(cfg.B):
        d = int(wl.divergence[b])
        assert len(ix.match(wl.probe(b))) == d // P, b
    for p in prefix_pages:
        assert pool.refcount(int(p)) == cfg.B + 1


@pytest.mark.parametrize("seed", range(5))
def test_prefix_index_matches_brute_force_model(seed):
    rng = np.random.default_rng(100 + seed)
    P, n = 4, 48
    order = rng.permutation(n).astype(np.int32)
    pool, mpool = K.KvPool(n, P, order), PoolModel(n, P, order)
    ix, mix = K.KvPrefixIndex(P, salt=7), PrefixModel(P, salt=7)
    vocab = 3  # tiny vocabulary: many shared prefixes and collisions of blocks
    seqs = []
    for it in range(120):
        op = rng.integers(0, 5)
        if op <= 1:  # new sequence: match, share, allocate the rest, register
            L = int(rng.integers(1, 6 * P))
            toks = list(rng.integers(0, vocab, L))
            hit, mhit = ix.match(toks), mix.match(toks)
            assert list(hit) == mhit
            need = -(-L // P) - len(hit)
            try:
                mpool.incref(mhit)
                new_m = mpool.alloc(need)
            except PoolError as e:
                with pytest.raises(K.KvError) as ei:
                    pool.incref(hit)
                    pool.alloc(need)
                assert ei.value.name == e.kind
                if e.kind == "OOM":
                    pool.free(hit)
                    mpool.free_pages(mhit)
                continue
            pool.incref(hit)
            new = pool.alloc(need)
            assert list(new) == new_m
            pages = list(hit) + list(new)
            ix.register(pool, toks, pages)
            mix.register(mpool, toks, pages)
            seqs.append((toks, pages))
        elif op == 2 and seqs:  # a sequence finishes
            toks, pages = seqs.pop(int(rng.integers(0, len(seqs))))
            pool.free(pages)
            mpool.free_pages(pages)
        else:  # probe
            L = int(rng.integers(0, 6 * P))
            toks = list(rng.integers(0, vocab, L))
            assert list(ix.match(toks)) == mix.match(toks)
        assert ix.num_entries() == len(mix.entries)
        assert pool.num_free() == mpool.num_free()


def test_prefix_register_errors():
    P = 4
    pool = K.KvPool(8, P)
    ix = K.KvPrefixIndex(P)
    a = pool.alloc(2)
    ix.register(pool, list(range(8)), a)
    with pytest.raises(K.KvError) as e:  # page already holds another prefix
        ix.register(pool, list(range(10, 18)), a)
    assert e.value.name == "ARG"
    with pytest.raises(K.KvError) as e:  # page not allocated
        ix.register(pool, list(range(20, 24)), [7])
    assert e.value.name == "BAD_ID"
    other = K.KvPool(8, 8)
    with pytest.raises(K.KvError):  # page size differs
        ix.register(other, list(range(8)), [0])
    with pytest.raises(K.KvError):  # match with a different page size
        K.lib()
        import ctypes
        n = ctypes.c_int32()
        t = np.arange(8, dtype=np.int32)
        K._check("kv_prefix_match", K.lib().kv_prefix_match(ix._h, t.ctypes.data, 8, 8, None, n))


def test_salt_separates_identities():
    P = 4
    pool = K.KvPool(8, P)
    ix_a, ix_b = K.KvPrefixIndex(P, salt=1), K.KvPrefixIndex(P, salt=2)
    toks = list(range(8))
    pages = pool.alloc(2)
    ix_a.register(pool, toks, pages)
    assert len(ix_a.match(toks)) == 2 and len(ix_b.match(toks)) == 0


# ------------------------------------------------------------------ device entry points: checks only
def test_device_entry_argument_checks_without_gpu():
    L = K.lib()
    # explicit split counts need no device query
    assert K.paged_decode_num_splits(4, 8, 100, 16, 3) == 3
    assert K.paged_decode_num_splits(4, 8, 10, 16, 64) == 10
    assert K.paged_decode_workspace_bytes(2, 32, 8, 128, 64, 16, 1) == 0
    S = K.paged_decode_num_splits(2, 8, 64, 16, 4)
    assert K.paged_decode_workspace_bytes(2, 32, 8, 128, 64, 16, 4) == 2 * 32 * S * (128 * 4 + 8)
    # unsupported shapes are refused before any launch
    args = [None] * 4 + [None, 16, None, 2, 32, 8, 96, 16, 64, 0.1, 1, 1, None, 0, None, None]
    assert L.paged_decode_attention(*args) == K.KV_ERR_UNSUPPORTED  # Dh = 96
    args[10] = 128
    args[11] = 24
    assert L.paged_decode_attention(*args) == K.KV_ERR_UNSUPPORTED  # page size 24
    args[11] = 16
    args[8], args[9] = 65, 1
    assert L.paged_decode_attention(*args) == K.KV_ERR_UNSUPPORTED  # GQA group of 65 (tensor-core limit 64)
    args[8] = 33
    K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_SIMT)
    try:
        assert L.paged_decode_attention(*args) == K.KV_ERR_UNSUPPORTED  # CUDA-core limit 32
    finally:
        K.paged_decode_set_kernel(K.KV_DECODE_KERNEL_AUTO)
    assert L.paged_decode_set_kernel(7) == K.KV_ERR_ARG
    args[8], args[9] = 32, 7
    assert L.paged_decode_attention(*args) == K.KV_ERR_ARG  # H_q % H_kv != 0
    args[9] = 8
    args[7] = 0
    assert L.paged_decode_attention(*args) == K.KV_OK  # B = 0: nothing to do
    args[7] = 2
    assert L.paged_decode_attention(*args) == K.KV_ERR_ARG  # null pointers
    assert L.kv_append(None, None, None, None, None, 0, 8, 128, 16, 10, 1, None, None) == K.KV_OK
    assert L.kv_append(None, None, None, None, None, 3, 8, 128, 16, 10, 1, None, None) == K.KV_ERR_ARG
    assert L.kv_append(None, None, None, None, None, 3, 8, 128, 16, 10, 9, None, None) == K.KV_ERR_ARG


def test_extension_entry_argument_checks_without_gpu():
    """E4M3, RoPE, fused and multi-token entry points refuse bad arguments before any CUDA call."""
    L = K.lib()
    # kv_append_fp8: source must be a 16/32-bit type, Dh a multiple of 16, scales and pointers present
    assert L.kv_append_fp8(None, None, None, None, 3, None, None, None, 2, 8, 128, 16, 10, None, None) == K.KV_ERR_ARG
    assert L.kv_append_fp8(None, None, None, None, 1, None, None, None, 2, 8, 120, 16, 10, None, None) == \
        K.KV_ERR_UNSUPPORTED
    assert L.kv_append_fp8(None, None, None, None, 1, None, None, None, 0, 8, 128, 16, 10, None, None) == K.KV_OK
    assert L.kv_append_fp8(None, None, None, None, 1, None, None, None, 2, 8, 128, 16, 10, None, None) == K.KV_ERR_ARG
    # paged_decode_attention_fp8: q must be bf16 / fp16, scales present
    fp8 = [None, None, 0, None, None, None, None, None, 16, None, 2, 32, 8, 128, 16, 64, 0.1, 0, None, 0, None, None]
    assert L.paged_decode_attention_fp8(*fp8) == K.KV_ERR_ARG  # q of fp32
    fp8[2] = 1
    assert L.paged_decode_attention_fp8(*fp8) == K.KV_ERR_ARG  # no scales
    # kv_rope_append: style, q / q_out pairing, row size
    rope = [None] * 9 + [64, 0, 2, 32, 8, 128, 16, 10, 1, None, None]
    rope[9] = 64
    assert L.kv_rope_append(*rope) == K.KV_ERR_ARG  # null pointers
    rope[10] = 5
    assert L.kv_rope_append(*rope) == K.KV_ERR_ARG  # unknown pairing
    rope[10] = 0
    rope[14] = 8
    assert L.kv_rope_append(*rope) == K.KV_ERR_UNSUPPORTED  # 16-byte rows cannot hold vector pairs
    rope[14], rope[11] = 128, 0
    assert L.kv_rope_append(*rope) == K.KV_OK  # no tokens
    # fused rotate + append + decode: 16-bit K/V only, table required
    fused = [None] * 7 + [16, None, None, 64, 0, 2, 32, 8, 128, 16, 64, 0.1, 0, 0, None, 0, None, None]
    assert L.paged_decode_attention_rope_append(*fused) == K.KV_ERR_UNSUPPORTED  # fp32 K/V
    fused[19] = 1
    assert L.paged_decode_attention_rope_append(*fused) == K.KV_ERR_ARG  # no k_new / table
    # multi-token query: fp32 unsupported, shapes checked, nothing to do for empty batches
    pre = [None, None, None, 16, None, None, None, 8, None, 2, 32, 8, 128, 16, 64, 0.1, 0, None, None]
    assert L.paged_prefill_attention(*pre) == K.KV_ERR_UNSUPPORTED  # fp32
    pre[16] = 1
    pre[12] = 96
    assert L.paged_prefill_attention(*pre) == K.KV_ERR_UNSUPPORTED  # Dh = 96
    pre[12] = 128
    pre[10] = 130
    assert L.paged_prefill_attention(*pre) == K.KV_ERR_ARG  # H_q % H_kv != 0
    pre[10] = 32
    pre[3] = 0
    assert L.paged_prefill_attention(*pre) == K.KV_OK  # no chunk rows
    pre[3] = 16
    assert L.paged_prefill_attention(*pre) == K.KV_ERR_ARG  # null pointers


# ------------------------------------------------------------------ copy-on-write vs model
@pytest.mark.parametrize("seed", range(4))
def test_cow_tails_matches_model(seed):
    rng = np.random.default_rng(500 + seed)
    P, n, max_blocks = 4, 64, 8
    order = rng.permutation(n).astype(np.int32)
    pool, model = K.KvPool(n, P, order), PoolModel(n, P, order)
    B = 6
    tab = np.full((B, max_blocks), -1, np.int32)
    mtab = [[-1] * max_blocks for _ in range(B)]
    lens = np.zeros(B, np.int32)
    for b in range(B):
        if b > 0 and rng.random() < 0.5:  # fork of an earlier sequence
            src = int(rng.integers(0, b))
            ids = [int(x) for x in tab[src] if x >= 0]
            pool.incref(ids)
            model.incref(ids)
            tab[b] = tab[src]
            mtab[b] = list(mtab[src])
            lens[b] = lens[src]
        else:
            L = int(rng.integers(1, max_blocks * P - 1))
            k = -(-L // P)
            ids = pool.alloc(k)
            assert list(ids) == model.alloc(k)
            tab[b, :k] = ids
            mtab[b][:k] = list(ids)
            lens[b] = L
    src, dst = pool.cow_tails(tab, lens)
    pairs = model.cow_tails(mtab, max_blocks, [int(x) for x in lens])
    assert list(zip(src.tolist(), dst.tolist())) == pairs
    assert tab.tolist() == mtab
    for p in range(n):
        assert pool.refcount(p) == model.refcount(p)
    assert pool.num_free() == model.num_free()
    # afterwards every append goes to a private page
    pool.append_slots(tab, lens.copy())


def test_cow_tails_oom_leaves_everything_unchanged():
    pool = K.KvPool(2, 4)
    a = pool.alloc(2)
    pool.incref(a[1:])
    tab = np.array([[a[0], a[1]], [a[0], a[1]]], np.int32)
    pool.incref(a[:1])
    before = tab.copy()
    with pytest.raises(K.KvError) as e:
        pool.cow_tails(tab, np.array([6, 6], np.int32))
    assert e.value.name == "OOM" and np.array_equal(tab, before) and pool.refcount(a[1]) == 2
