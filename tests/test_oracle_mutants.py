"""The oracle's pins must catch plausible mistakes in it.

Each case plants one mistake in a private copy of the C oracle (a dropped
term, a wrong sign or index, a transposed operand), builds that copy on the
CPU, and checks that at least one of the pin checks below fails on it, while
the unmodified source passes them all.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

from helpers import ROOT, golden
from oracle import reference as R
from paged_kv_cache_433_b200 import workloads as W

SRC = os.path.join(ROOT, "oracle", "decode_ref.c")

MUTANTS = {
    "block index uses offset": ("block_tables[(int64_t)b * max_blocks + t / P];\n            if (page < 0",
                                "block_tables[(int64_t)b * max_blocks + t % P];\n            if (page < 0"),
    "offset uses block index": ("kvh) * P + (t % P)) * Dh;\n            double acc",
                                "kvh) * P + (t / P)) * Dh;\n            double acc"),
    "scale dropped": ("s[t] = scale * acc;", "s[t] = acc;"),
    "GQA head mapping modulo": ("int32_t kvh = h / g;", "int32_t kvh = h % g;"),
    "softmax exponent sign": ("s[t] = exp(s[t] - m);", "s[t] = exp(m - s[t]);"),
    "row maximum not subtracted": ("s[t] = exp(s[t] - m);", "s[t] = exp(s[t]);"),
    "values read from K": ("o[d] += p * elem(v_pages, row + d, dtype);", "o[d] += p * elem(k_pages, row + d, dtype);"),
    "normaliser dropped": ("double p = s[t] / l;", "double p = s[t];"),
    "query row of wrong head": ("elem(q, ((int64_t)b * H_q + h) * Dh + d, dtype)", "elem(q, ((int64_t)b * H_q + kvh) * Dh + d, dtype)"),
    "fp16 exponent bias": ("e - 25);", "e - 24);"),
    "bf16 shift": ("((uint32_t)h) << 16;", "((uint32_t)h) << 15;"),
    "last position dropped": ("for (int32_t t = 0; t < len && !bad; ++t)", "for (int32_t t = 0; t + 1 < len && !bad; ++t)"),
}


def _build(tmp_path, name, text):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(text)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(c), "-o", str(so), "-lm"], check=True)
    return str(so)


def _checks(monkeypatch, so_path):
    """Run the pin checks against the library at so_path; return the names that fail."""
    lib = ctypes.CDLL(so_path)
    saved = R._LIB
    R._LIB = None
    real = R._lib()
    for fn in ("oracle_paged_decode", "oracle_decode_storage"):
        f = getattr(lib, fn)
        f.restype = getattr(real, fn).restype
        f.argtypes = getattr(real, fn).argtypes
    lib.oracle_max_threads = real.oracle_max_threads
    monkeypatch.setattr(R, "_LIB", lib)
    failed = []

    def check(name, fn):
        try:
            if not fn():
                failed.append(name)
        except ValueError:  # the oracle reported an out-of-range access
            failed.append(name + " (error)")

    try:
        check("single-query", lambda: _single_query())
        check("fp16-decode", lambda: _fp16_decode())
        check("bf16-decode", lambda: _bf16_decode())
        for dt in ("bf16", "fp16"):
            check(f"causal-{dt}", lambda dt=dt: _causal(dt))
    finally:
        R._LIB = saved
    return failed


def _single_query():
    """The single-query example through the C decode, as given and shifted by +800.

    Softmax is unchanged when every score moves by the same constant, so the
    shifted case has the same answer; it overflows exp() unless the row
    maximum is subtracted first.
    """
    gd = golden("single_query_three_scores.json")
    for shift in (0.0, 800.0):
        kp = np.zeros((4, 1, 2, 2), np.float32)
        vp = np.zeros((4, 1, 2, 2), np.float32)
        tab = np.array([[3, 1]], np.int32)
        R.scatter_to_pages(kp, tab[0], np.array([[x + shift, 0.0] for x in gd["scores"]], np.float32)[:, None, :])
        R.scatter_to_pages(vp, tab[0], np.array(gd["values"], np.float32)[:, None, :])
        out = R.paged_decode(np.array([[[1.0, 0.0]]], np.float32), kp, vp, tab, np.array([3], np.int32), 1.0, "fp32")
        if not np.allclose(out[0, 0], [7.1025624236, 5.3447222869], atol=1e-9):
            return False
    return True


def _fp16_decode():
    """Storage decoding against numpy's float16."""
    bits = np.arange(0, 65536, 97, dtype=np.uint32).astype(np.uint16)
    lib16 = bits.view(np.float16).astype(np.float64)
    ok = ~np.isnan(lib16)
    return np.array_equal(R.decode_storage(bits, "fp16")[ok], lib16[ok])


def _bf16_decode():
    """bf16 decoding against the definition as the upper half of a float32 (numpy view)."""
    bits = np.arange(0, 65536, 97, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        libbf = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ok = ~np.isnan(libbf)
    return np.array_equal(R.decode_storage(bits, "bf16")[ok], libbf[ok])


def _causal(dt):
    """Incremental paged decode == full causal recompute (GQA, P=4)."""
    T, Hq, Hkv, Dh, P = 13, 4, 2, 8, 4
    Q = W.normal_storage(21, 1, (), (T, Hq, Dh), dt)
    K = W.normal_storage(21, 2, (), (T, Hkv, Dh), dt)
    V = W.normal_storage(21, 3, (), (T, Hkv, Dh), dt)
    full = R.causal_attention(*(R.decode_storage(x, dt) for x in (Q, K, V)), 0.35)
    perm = W.page_order(6, 21)
    for t in (1, 4, 5, 13):
        nb = -(-t // P)
        kp = np.zeros((6, Hkv, P, Dh), np.uint16)
        vp = np.zeros((6, Hkv, P, Dh), np.uint16)
        R.scatter_to_pages(kp, perm[:nb], K[:t])
        R.scatter_to_pages(vp, perm[:nb], V[:t])
        o = R.paged_decode(Q[t - 1][None], kp, vp, perm[:nb][None].astype(np.int32), np.array([t], np.int32), 0.35, dt)
        if not np.allclose(o[0], full[t - 1], atol=1e-9):
            return False
    return True


def test_unmodified_oracle_passes_all_checks(tmp_path, monkeypatch):
    so = _build(tmp_path, "orig", open(SRC).read())
    assert _checks(monkeypatch, so) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, monkeypatch, name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor not unique/not found: {name}"
    so = _build(tmp_path, "mutant", src.replace(old, new))
    assert _checks(monkeypatch, so), f"mutant survived: {name}"
