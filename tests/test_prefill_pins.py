"""Pins of the multi-token (chunked prefill) oracle: against the full causal
recompute on logical rows, the one-token case against decode, physical page
order; planted mistakes must fail a pin."""
import importlib.util
import os

import numpy as np
import pytest

from helpers import ROOT
from oracle import reference as R
from paged_kv_cache_433_b200 import workloads as W

CFG = W.DecodeConfig("prefill-pin", "bf16", B=3, H_q=4, H_kv=2, Dh=32, page_size=4, seed=70)
LENS = [11, 6, 9]      # total lengths after the chunk is appended
CHUNK = [5, 6, 1]      # chunk rows per sequence (the second is a whole prompt)


def _setup(order_seed=0):
    P = CFG.page_size
    pages = [-(-L // P) for L in LENS]
    num_pages = sum(pages) + 2
    perm = W.generator(71, W.S_PAGES, order_seed).permutation(num_pages)
    tab = np.full((CFG.B, max(pages)), -1, np.int32)
    k = 0
    for b, n in enumerate(pages):
        tab[b, :n] = perm[k:k + n]
        k += n
    kp = np.full((num_pages, CFG.H_kv, P, CFG.Dh), 0x7FC0, np.uint16)
    vp = kp.copy()
    logical = []
    for b, L in enumerate(LENS):
        kr, vr = W.kv_rows(CFG, 0, b, L)
        R.scatter_to_pages(kp, tab[b], kr)
        R.scatter_to_pages(vp, tab[b], vr)
        logical.append((kr, vr))
    q_start = np.concatenate([[0], np.cumsum(CHUNK)]).astype(np.int32)
    q = np.concatenate([W.all_queries(CFG, 0, b, L)[L - n:] for b, (L, n) in enumerate(zip(LENS, CHUNK))])
    return q, q_start, kp, vp, tab, logical


def _check_causal(mod):
    q, qs, kp, vp, tab, logical = _setup()
    got = mod.paged_prefill(q, qs, kp, vp, tab, LENS, CFG.scale, "bf16")
    for b, (L, n) in enumerate(zip(LENS, CHUNK)):
        Q = R.decode_storage(W.all_queries(CFG, 0, b, L), "bf16")
        Kl, Vl = (R.decode_storage(x, "bf16") for x in logical[b])
        full = R.causal_attention(Q, Kl, Vl, CFG.scale)  # every position of the sequence
        assert np.allclose(got[qs[b]:qs[b + 1]], full[L - n:], atol=1e-12, rtol=1e-12), f"sequence {b}"


def _check_single(mod):
    q, qs, kp, vp, tab, _ = _setup()
    one = np.array([0, 1], np.int32)
    row = q[qs[0] + CHUNK[0] - 1:qs[0] + CHUNK[0]]  # the last chunk row of sequence 0 = its decode query
    got = mod.paged_prefill(row, one, kp, vp, tab[:1], LENS[:1], CFG.scale, "bf16")
    ref = R.paged_decode(row, kp, vp, tab[:1], np.array(LENS[:1], np.int32), CFG.scale, "bf16")
    assert np.array_equal(got, ref)


def _check_pages(mod):
    a = _setup(0)
    b = _setup(1)
    ga = mod.paged_prefill(a[0], a[1], a[2], a[3], a[4], LENS, CFG.scale, "bf16")
    gb = mod.paged_prefill(b[0], b[1], b[2], b[3], b[4], LENS, CFG.scale, "bf16")
    assert np.allclose(ga, gb, atol=1e-13, rtol=0)


def test_prefill_matches_full_causal_recompute():
    _check_causal(R)


def test_one_token_chunk_is_decode():
    _check_single(R)


def test_prefill_independent_of_physical_page_order():
    _check_pages(R)


def test_positions_of_chunk_rows():
    assert R.chunk_positions([0, 3, 5, 5], [10, 2, 7]).tolist() == [7, 8, 9, 0, 1]


PREFILL_MUTANTS = {
    "chunk starts one late": ("pos[qs[b]:qs[b + 1]] = sl[b] - n + np.arange(n)",
                              "pos[qs[b]:qs[b + 1]] = sl[b] - n + 1 + np.arange(n)"),
    "row does not see itself": ("lens = (pos + 1).astype(np.int32)", "lens = np.maximum(pos, 1).astype(np.int32)"),
    "table of the wrong sequence": ("owner = np.repeat(np.arange(B), np.diff(qs))",
                                    "owner = np.repeat(np.arange(B)[::-1], np.diff(qs))"),
}


def _load_mutant(tmp_path, old, new):
    src = open(os.path.join(ROOT, "oracle", "reference.py"), encoding="utf-8").read()
    assert old in src
    path = tmp_path / "reference_mut.py"
    path.write_text(src.replace(old, new).replace("from . import build_oracle", "from oracle import build_oracle"))
    spec = importlib.util.spec_from_file_location("reference_mut", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", sorted(PREFILL_MUTANTS))
def test_prefill_mutant_is_caught(tmp_path, name):
    mod = _load_mutant(tmp_path, *PREFILL_MUTANTS[name])
    failed = 0
    for check in (_check_causal, _check_single, _check_pages):
        try:
            check(mod)
        except (AssertionError, ValueError):
            failed += 1
    assert failed, f"mutant '{name}' survived every pin"
