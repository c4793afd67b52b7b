"""Pins for the CPU oracle: values the pages print, closed forms, invariants.

These tests never touch the CUDA path. Every expected value is either printed
on a page (fixtures under tests/golden/, each with its source) or fixed by
mathematics independently of the oracle's code path.
"""
import math

import numpy as np
import pytest
import torch

from helpers import golden
from oracle import reference as R
from oracle.pool_model import PoolModel, PrefixModel, PoolError
from paged_kv_cache_433_b200 import workloads as W


# ---------------------------------------------------------------- online merge
def test_online_merge_two_blocks_printed_values():
    gd = golden("online_merge_two_blocks.json")
    blocks = [(b["scores"], np.array(b["values"])) for b in gd["blocks"]]
    st1 = R.merge_block(None, *blocks[0])
    assert st1[0] == gd["after_block_1"]["m"] and st1[1] == gd["after_block_1"]["l"]
    assert st1[2][0] == gd["after_block_1"]["u"]
    m, l, u, o = R.online_softmax(blocks)
    tol = 0.5 * 10.0 ** (-gd["printed_decimals"])
    assert m == 3.0
    assert abs(l - gd["l"]) <= tol
    assert abs(u[0] - gd["u"]) <= tol
    assert abs(o[0] - gd["o"]) <= tol
    assert round(o[0], 4) == gd["o_short"]
    # the page's statement: equal to a full softmax over [1, 3] then weighting
    assert abs(R.softmax_weighted_sum([1.0, 3.0], np.array([2.0, 10.0]))[0] - gd["o"]) <= tol


def test_online_merge_counter_example_is_wrong():
    gd = golden("online_merge_two_blocks.json")
    blocks = [(b["scores"], np.array(b["values"])) for b in gd["blocks"]]
    _, _, _, o_bad = R.online_softmax(blocks, rescale_old=False)
    assert abs(o_bad[0] - gd["o"]) > 0.1


def test_single_query_closed_form_and_order_invariance():
    gd = golden("single_query_three_scores.json")
    s = gd["scores"]
    v = np.array(gd["values"])
    # closed form: weights e^0, e^2, e^1 over their sum
    w = [math.exp(0.0), math.exp(2.0), math.exp(1.0)]
    want = [(w[0] * 5 + w[1] * 10 + w[2] * 0) / sum(w), (w[0] * 5 + w[1] * 0 + w[2] * 20) / sum(w)]
    assert want[0] == pytest.approx(7.1025624236, abs=1e-9)
    assert want[1] == pytest.approx(5.3447222869, abs=1e-9)
    for perm in ([0, 1, 2], [2, 0, 1], [1, 2, 0], [2, 1, 0]):
        blocks = [([s[i]], v[i:i + 1]) for i in perm]
        _, _, _, o = R.online_softmax(blocks)
        assert np.allclose(o, want, atol=1e-12, rtol=0)
    # intermediate states in read order C/A/B
    st = R.merge_block(None, [s[0]], v[0:1])
    assert st[0] == 0.0 and st[1] == 1.0 and np.allclose(st[2] / st[1], [5, 5])
    st = R.merge_block(st, [s[1]], v[1:2])
    assert st[0] == 2.0 and st[1] == pytest.approx(1.0 + math.exp(-2.0))
    assert np.allclose(st[2] / st[1], [(math.exp(-2) * 5 + 10) / (1 + math.exp(-2)), math.exp(-2) * 5 / (1 + math.exp(-2))])


def test_single_query_through_paged_c_oracle():
    """The same example through the fp64 C decode: q=[1,0], K rows put the scores in dim 0, scale 1."""
    gd = golden("single_query_three_scores.json")
    s, v = gd["scores"], np.array(gd["values"], dtype=np.float32)
    P, H, Dh = 2, 1, 2
    k_pages = np.zeros((4, H, P, Dh), np.float32)
    v_pages = np.full((4, H, P, Dh), np.nan, np.float32)
    table = np.array([[3, 1]], np.int32)
    K = np.array([[x, 0.0] for x in s], np.float32)[:, None, :]
    R.scatter_to_pages(k_pages, table[0], K)
    R.scatter_to_pages(v_pages, table[0], v[:, None, :])
    q = np.array([[[1.0, 0.0]]], np.float32)
    out = R.paged_decode(q, k_pages, v_pages, table, np.array([3], np.int32), 1.0, "fp32")
    assert np.allclose(out[0, 0], [7.1025624236, 5.3447222869], atol=1e-9, rtol=0)
    # softmax does not change when all scores move by one constant; +800 would
    # overflow exp() unless the row maximum is subtracted first
    R.scatter_to_pages(k_pages, table[0], K + np.array([800.0, 0.0], np.float32))
    out = R.paged_decode(q, k_pages, v_pages, table, np.array([3], np.int32), 1.0, "fp32")
    assert np.allclose(out[0, 0], [7.1025624236, 5.3447222869], atol=1e-9, rtol=0)


# ---------------------------------------------------- decode vs full causal recompute
def _paged_pool(rows_k, rows_v, P, num_pages, perm, dtype_store):
    T = rows_k.shape[0]
    nblk = -(-T // P)
    table = np.asarray(perm[:nblk], np.int32)
    fill = np.float32(np.nan) if dtype_store == np.float32 else np.uint16(0x7FC0)
    kp = np.full((num_pages, rows_k.shape[1], P, rows_k.shape[2]), fill, dtype=dtype_store)
    vp = np.full_like(kp, fill)
    R.scatter_to_pages(kp, table, rows_k)
    R.scatter_to_pages(vp, table, rows_v)
    return kp, vp, table


@pytest.mark.parametrize("dtype", ["fp32", "bf16", "fp16"])
@pytest.mark.parametrize("P,H_q,H_kv", [(4, 4, 2), (16, 4, 2), (3, 2, 2), (5, 6, 1)])
def test_incremental_decode_equals_full_causal(dtype, P, H_q, H_kv):
    """Cached incremental decode (append, then attend) == rows of full causal attention.

    "07｜KV Cache、FlashAttention与PagedAttention的内部过程" Q025 (old K/V do not
    change when a token is appended; the new token attends to all cached K/V).
    """
    T, Dh = 37, 8
    seed = 11
    Q = W.normal_storage(seed, 1, (P, H_q), (T, H_q, Dh), dtype)
    K = W.normal_storage(seed, 2, (P, H_q), (T, H_kv, Dh), dtype)
    V = W.normal_storage(seed, 3, (P, H_q), (T, H_kv, Dh), dtype)
    Qd, Kd, Vd = (R.decode_storage(x, dtype) for x in (Q, K, V))
    scale = 1.0 / math.sqrt(Dh)
    full = R.causal_attention(Qd, Kd, Vd, scale)
    num_pages = -(-T // P) + 3
    perm = W.page_order(num_pages, seed, P)
    store = np.float32 if dtype == "fp32" else np.uint16
    for t in range(1, T + 1):
        kp, vp, table = _paged_pool(K[:t], V[:t], P, num_pages, perm, store)
        out = R.paged_decode(Q[t - 1][None], kp, vp, table[None], np.array([t], np.int32), scale, dtype)
        assert np.allclose(out[0], full[t - 1], atol=1e-12, rtol=1e-12), t


def test_page_permutation_invariance_exact():
    """Same logical content behind two different physical permutations -> identical output.

    "07｜KV Cache、FlashAttention与PagedAttention的内部过程" Q028: the block table
    changes where blocks are stored, not the logical token order.
    """
    cfg = W.TINY
    T, P = 77, 16
    K = W.normal_storage(5, 2, (0,), (T, cfg.H_kv, cfg.Dh), "bf16")
    V = W.normal_storage(5, 3, (0,), (T, cfg.H_kv, cfg.Dh), "bf16")
    q = W.normal_storage(5, 4, (0,), (1, cfg.H_q, cfg.Dh), "bf16")
    outs = []
    for s in (1, 2, 3):
        kp, vp, table = _paged_pool(K, V, P, 12, W.page_order(12, s), np.uint16)
        outs.append(R.paged_decode(q, kp, vp, table[None], np.array([T], np.int32), cfg.scale, "bf16"))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_special_cases_closed_forms():
    Dh, P = 16, 4
    rng = np.random.default_rng(0)
    V = rng.standard_normal((9, 1, Dh)).astype(np.float32)
    K = rng.standard_normal((9, 1, Dh)).astype(np.float32)
    q = rng.standard_normal((1, 1, Dh)).astype(np.float32)
    # seq_len 1 -> exactly V_0
    kp, vp, table = _paged_pool(K[:1], V[:1], P, 4, [2, 0, 1, 3], np.float32)
    out = R.paged_decode(q, kp, vp, table[None], np.array([1], np.int32), 0.25, "fp32")
    assert np.array_equal(out[0, 0], V[0, 0].astype(np.float64))
    # all keys equal -> uniform weights -> mean of V
    Ke = np.repeat(K[:1], 9, axis=0)
    kp, vp, table = _paged_pool(Ke, V, P, 4, [2, 0, 1, 3], np.float32)
    out = R.paged_decode(q, kp, vp, table[None], np.array([9], np.int32), 0.25, "fp32")
    assert np.allclose(out[0, 0], V[:, 0].astype(np.float64).mean(axis=0), atol=1e-12)
    # seq_len 0 -> zeros
    out = R.paged_decode(q, kp, vp, table[None], np.array([0], np.int32), 0.25, "fp32")
    assert np.array_equal(out, np.zeros_like(out))


def test_gqa_equals_mha_with_repeated_heads():
    """GQA (H_q=4, H_kv=2) equals MHA whose KV heads are repeated: head h uses KV head h // 2."""
    T, Dh, P = 21, 8, 4
    K = W.normal_storage(8, 2, (0,), (T, 2, Dh), "fp16")
    V = W.normal_storage(8, 3, (0,), (T, 2, Dh), "fp16")
    q = W.normal_storage(8, 4, (0,), (1, 4, Dh), "fp16")
    perm = W.page_order(8, 8)
    kp, vp, table = _paged_pool(K, V, P, 8, perm, np.uint16)
    gqa = R.paged_decode(q, kp, vp, table[None], np.array([T], np.int32), 0.3, "fp16")
    K4, V4 = np.repeat(K, 2, axis=1), np.repeat(V, 2, axis=1)
    kp4, vp4, table4 = _paged_pool(K4, V4, P, 8, perm, np.uint16)
    mha = R.paged_decode(q, kp4, vp4, table4[None], np.array([T], np.int32), 0.3, "fp16")
    assert np.array_equal(gqa, mha)
    # and each head against the logical (unpaged) definition
    ref = R.decode_logical(R.decode_storage(q[0], "fp16"), R.decode_storage(K, "fp16"), R.decode_storage(V, "fp16"), 0.3)
    assert np.allclose(gqa[0], ref, atol=1e-12)


def test_storage_decoding_matches_library_casts():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f16 = R.decode_storage(bits, "fp16")
    lib16 = bits.view(np.float16).astype(np.float64)
    assert np.array_equal(np.isnan(f16), np.isnan(lib16))
    ok = ~np.isnan(lib16)
    assert np.array_equal(f16[ok], lib16[ok])
    bf = R.decode_storage(bits, "bf16")
    libbf = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(np.isnan(bf), np.isnan(libbf))
    ok = ~np.isnan(libbf)
    assert np.array_equal(bf[ok], libbf[ok])


# ---------------------------------------------------------------- paging arithmetic
def test_block_table_worked_example():
    gd = golden("block_table_example.json")
    P, table = gd["page_size"], gd["table"]
    lk = gd["lookup"]
    assert R.logical_block(lk["pos"], P) == (lk["logical_block"], lk["offset"])
    assert R.physical_slot(table, P, lk["pos"]) == lk["physical_page"] * P + lk["offset"]
    for a in gd["appends"]:
        assert R.physical_slot(table, P, a["pos"]) == a["page"] * P + a["offset"]
        assert not R.needs_new_page(a["pos"], P)
    assert R.needs_new_page(gd["first_position_needing_new_block"], P)
    # the same walk through the pool model: blocks 7, 2, 19 handed out first
    order = [7, 2, 19] + [i for i in range(24) if i not in (7, 2, 19)]
    pool = PoolModel(24, P, order)
    tab = [pool.alloc(3) + [-1, -1]]
    assert tab[0][:3] == table
    lens = [gd["cached_len"]]
    s10 = pool.append_slots(tab, 5, lens)
    s11 = pool.append_slots(tab, 5, lens)
    assert (s10, s11) == ([19 * P + 2], [19 * P + 3])
    free_before = pool.num_free()
    s12 = pool.append_slots(tab, 5, lens)
    assert pool.num_free() == free_before - 1 and tab[0][3] == order[3] and s12 == [order[3] * P]


def test_fragmentation_example():
    gd = golden("fragmentation.json")
    assert R.blocks_for_len(gd["length"], gd["page_size"]) == (gd["blocks"], gd["slots"], gd["wasted"])
    assert R.blocks_for_len(0, 16) == (0, 0, 0)
    assert R.blocks_for_len(16, 16) == (1, 16, 0)
    assert R.blocks_for_len(17, 16) == (2, 32, 15)


def test_kv_bytes_formula():
    for c in golden("kv_bytes.json")["cases"]:
        tot = R.kv_cache_bytes(c["L"], c["B"], c["T"], c["H_kv"], c["Dh"], c["bytes"])
        assert tot == c["total_bytes"], c["source"]
        if "per_token_bytes" in c:
            assert R.kv_cache_bytes(c["L"], c["B"], 1, c["H_kv"], c["Dh"], c["bytes"]) == c["per_token_bytes"]
            assert c["L"] * c["B"] * c["T"] * c["H_kv"] * c["Dh"] == c["k_elements"]
            assert tot // 2 == c["k_bytes"]
    assert R.kv_cache_bytes_ragged(32, [8192], 8, 128, 2) == 2 ** 30
    assert R.kv_cache_bytes_ragged(32, [8192] * 8, 8, 128, 2) == 8 * 2 ** 30


def test_token_count_context_example():
    gd = golden("token_counts.json")
    p, n = gd["prompt"], gd["generated"]
    assert sum(range(p, p + n)) == gd["positions_without_cache"]
    assert p + (n - 1) == gd["positions_with_cache"]
    assert round(gd["positions_without_cache"] / gd["positions_with_cache"] / 10) * 10 == gd["ratio_about"]


# ---------------------------------------------------------------- pool + prefix model
def _ids(s):
    return [ord(c) for c in s]


def test_prefix_demo():
    gd = golden("prefix_demo.json")
    P = gd["page_size_reading"]
    pool = PoolModel(16, P)
    ix = PrefixModel(P)
    cached = _ids(gd["cached"])
    pages = pool.alloc(3)
    ix.register(pool, cached, pages)
    req = _ids(gd["request"])
    lcp = next(i for i, (a, b) in enumerate(zip(cached, req)) if a != b)
    assert lcp == gd["shared_tokens"]
    hit = ix.match(req)
    assert len(hit) * P == gd["reusable_tokens"] and hit == pages[:1]
    assert len(req) - len(hit) * P == gd["recompute_at_least"]
    assert ix.match(_ids(gd["edit_at_start"]["request"])) == []
    # any other page size reproduces neither the 4 nor the 8 of the demo
    for P2 in (2, 3, 5, 6):
        assert (lcp // P2) * P2 != gd["reusable_tokens"]


def test_edit_invalidation_floors_to_page():
    gd = golden("edit_invalidation.json")
    P = 16
    toks = list(W.generator(3, 8).integers(0, W.VOCAB, 300))
    pool = PoolModel(64, P)
    ix = PrefixModel(P)
    ix.register(pool, toks, pool.alloc(300 // P + 1))
    edited = list(toks)
    edited[gd["edited_position"]] += 1
    assert len(ix.match(edited)) == gd["edited_position"] // P
    assert len(ix.match(toks)) == 300 // P


def test_refcount_shared_page_survives_one_free():
    pool = PoolModel(4, 16, [3, 1, 0, 2])
    a = pool.alloc(2)
    assert a == [3, 1]
    pool.incref([a[0]])  # second sequence shares block 3
    pool.free_pages(a)  # first sequence finishes
    assert pool.refcount(3) == 1 and 3 not in pool.free and list(pool.free) == [0, 2, 1]
    pool.free_pages([3])
    assert pool.refcount(3) == 0 and list(pool.free) == [0, 2, 1, 3]


def test_pool_errors_all_or_nothing():
    pool = PoolModel(3, 16)
    with pytest.raises(PoolError) as e:
        pool.alloc(4)
    assert e.value.kind == "OOM" and pool.num_free() == 3
    ids = pool.alloc(2)
    with pytest.raises(PoolError) as e:
        pool.free_pages([ids[0], ids[0]])
    assert e.value.kind == "DOUBLE_FREE" and pool.refcount(ids[0]) == 1
    with pytest.raises(PoolError) as e:
        pool.free_pages([7])
    assert e.value.kind == "BAD_ID"
    with pytest.raises(PoolError) as e:
        pool.incref([2])  # free and never registered
    assert e.value.kind == "BAD_ID"


def test_shared_tail_needs_copy_on_write():
    pool = PoolModel(8, 4)
    t = pool.alloc(1)
    pool.incref(t)  # two sequences hold the same partial block
    tabs = [[t[0], -1], [t[0], -1]]
    with pytest.raises(PoolError) as e:
        pool.append_slots(tabs, 2, [2, 2])
    assert e.value.kind == "SHARED_TAIL"
    # a full shared block is fine: the append opens a fresh block
    slots = pool.append_slots(tabs, 2, [4, 4])
    assert tabs[0][1] != tabs[1][1] and slots == [tabs[0][1] * 4, tabs[1][1] * 4]


def test_cached_free_page_is_matchable_until_reallocated():
    P = 4
    pool = PoolModel(4, P, [0, 1, 2, 3])
    ix = PrefixModel(P)
    toks = list(range(100, 112))
    pages = pool.alloc(3)
    ix.register(pool, toks, pages)
    pool.free_pages(pages)
    assert ix.match(toks) == pages  # cached but free
    pool.incref(pages[:2])  # prefix hit revives two blocks
    assert pool.refcount(0) == 1 and list(pool.free) == [3, 2]
    got = pool.alloc(1)  # hands out block 3 (never registered)
    assert got == [3] and ix.match(toks) == pages
    got = pool.alloc(1)  # hands out block 2 -> its prefix entry is dropped
    assert got == [2] and ix.match(toks) == pages[:2]


def test_merge_of_summarised_blocks_equals_full_softmax():
    """Merging per-block (m, l, u) summaries (the split combine rule) == online merge == full softmax."""
    gd = golden("online_merge_two_blocks.json")
    b1, b2 = ((b["scores"], np.array(b["values"])) for b in gd["blocks"])
    m, l, u = R.merge_states(R.block_state(*b1), R.block_state(*b2))
    assert m == 3.0 and abs(l - gd["l"]) <= 5e-7 and abs(u[0] - gd["u"]) <= 5e-7
    rng = np.random.default_rng(3)
    s = rng.standard_normal(40) * 3
    v = rng.standard_normal((40, 5))
    cuts = [0, 7, 8, 23, 40]
    states = [R.block_state(s[a:b], v[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
    acc = states[0]
    for st in states[1:]:
        acc = R.merge_states(acc, st)
    full = R.softmax_weighted_sum(s, v)
    assert np.allclose(acc[2] / acc[1], full, atol=1e-12)
    _, _, _, o = R.online_softmax([(s[a:b], v[a:b]) for a, b in zip(cuts[:-1], cuts[1:])])
    assert np.allclose(o, full, atol=1e-12)


def test_copy_on_write_of_a_shared_partial_tail():
    """[HB-07] Q028 table step 6: A and B share an unfilled last block; before
    they append different tokens one of them needs its own copy."""
    P = 4
    pool = PoolModel(16, P, list(range(16)))
    a = pool.alloc(3)  # 10 tokens: blocks 0, 1 full, block 2 holds positions 8, 9
    pool.incref(a)  # B is a fork of A (beam): shares all three blocks
    tabs = [a + [-1], list(a) + [-1]]
    lens = [10, 10]
    with pytest.raises(PoolError) as e:
        pool.append_slots([list(r) for r in tabs], 4, list(lens))
    assert e.value.kind == "SHARED_TAIL"
    pairs = pool.cow_tails(tabs, 4, lens)
    assert pairs == [(a[2], 3)]  # A copies, B (last holder) keeps the original
    assert tabs[0][:3] == [a[0], a[1], 3] and tabs[1][:3] == a
    assert pool.refcount(a[2]) == 1 and pool.refcount(3) == 1 and pool.refcount(a[0]) == 2
    slots = pool.append_slots(tabs, 4, lens)
    assert slots == [3 * P + 2, a[2] * P + 2]  # different physical slots, same logical position 10
    # full shared blocks are never copied; nothing to do once tails are private
    assert pool.cow_tails(tabs, 4, lens) == []


def test_copy_on_write_keeps_outside_holders():
    P = 4
    pool = PoolModel(16, P)
    a = pool.alloc(1)
    pool.incref(a)
    pool.incref(a)  # three holders; two of them append this step
    tabs = [[a[0], -1], [a[0], -1]]
    pairs = pool.cow_tails(tabs, 2, [2, 2])
    assert len(pairs) == 2 and pool.refcount(a[0]) == 1  # the third holder keeps the original
    with pytest.raises(PoolError) as e:
        PoolModel(1, P).cow_tails([[0]], 1, [4])  # full table row
    assert e.value.kind == "ARG"
