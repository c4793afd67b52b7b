"""Pins of the rotary-embedding oracle (oracle/rope.py) against values and
properties that do not come from the oracle itself, plus planted mistakes that
the pins must catch."""
import importlib.util
import math
import os

import numpy as np
import pytest
import torch

from helpers import ROOT
from oracle import rope as RP
from paged_kv_cache_433_b200 import workloads as W


# ---------------------------------------------------------------- rounding helpers vs torch's casts
def test_bf16_rounding_matches_torch_cast_including_ties():
    g = W.generator(31, W.S_Q)
    x = g.standard_normal(20000).astype(np.float32) * np.float32(3.0)
    bits = x.view(np.uint32).copy()
    bits[:2000] = (bits[:2000] & 0xFFFF0000) | 0x8000  # exact ties: even and odd upper halves
    bits[2000:2100] = (bits[2000:2100] & 0xFFFF0000) | 0x7FFF
    x = bits.view(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(RP.f32_to_bf16_bits(x), ref)


def test_fp16_rounding_matches_torch_cast():
    g = W.generator(32, W.S_Q)
    x = (g.standard_normal(20000) * 50).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(RP.to_storage(x, "fp16"), ref)


# ---------------------------------------------------------------- worked example (hand values)
def test_worked_example_dh4_base100():
    # Dh = 4, base = 100: theta_0 = 1, theta_1 = 100^(-1/2) = 0.1. Position 1, x = [1, 2, 3, 4].
    c1, s1 = 0.5403023058681398, 0.8414709848078965  # cos 1, sin 1
    c01, s01 = 0.9950041652780258, 0.09983341664682815  # cos 0.1, sin 0.1
    x = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    half = RP.rotate_fp64(x, [1], 4, 100.0, "half")[0, 0]  # pairs (0, 2) and (1, 3)
    assert np.allclose(half, [1 * c1 - 3 * s1, 2 * c01 - 4 * s01, 3 * c1 + 1 * s1, 4 * c01 + 2 * s01], atol=1e-15)
    inter = RP.rotate_fp64(x, [1], 4, 100.0, "interleaved")[0, 0]  # pairs (0, 1) and (2, 3)
    assert np.allclose(inter, [1 * c1 - 2 * s1, 2 * c1 + 1 * s1, 3 * c01 - 4 * s01, 4 * c01 + 3 * s01], atol=1e-15)
    tab = RP.rope_table(2, 4, 100.0)
    assert np.array_equal(tab[0], np.array([1, 1, 0, 0], np.float32))
    assert np.array_equal(tab[1], np.array([c1, c01, s1, s01], np.float32))


# ---------------------------------------------------------------- properties of the rotation
def _rand(seed, shape):
    return W.generator(seed, W.S_K).standard_normal(shape)


@pytest.mark.parametrize("style", RP.STYLES)
def test_relative_position_property(style):
    """<R(m) q, R(n) k> depends only on m - n (the reason the rotation is applied)."""
    Dh, base = 64, 10000.0
    q, k = _rand(1, (1, 1, Dh)), _rand(2, (1, 1, Dh))
    def dot(m, n):
        return float((RP.rotate_fp64(q, [m], Dh, base, style) * RP.rotate_fp64(k, [n], Dh, base, style)).sum())
    for m, n in [(5, 2), (103, 100), (7, 4), (2003, 2000)]:
        assert abs(dot(m, n) - dot(m - n, 0)) < 1e-10


@pytest.mark.parametrize("style", RP.STYLES)
def test_rotation_keeps_pair_norms_and_composes(style):
    Dh, base = 128, 500000.0
    x = _rand(3, (4, 2, Dh))
    pos = np.array([0, 1, 777, 32767])
    y = RP.rotate_fp64(x, pos, Dh, base, style)
    i, j = RP.pair_index(Dh, style)
    assert np.allclose(x[..., i] ** 2 + x[..., j] ** 2, y[..., i] ** 2 + y[..., j] ** 2, rtol=1e-12)
    assert np.array_equal(y[0], x[0])  # position 0 is the identity
    z = RP.rotate_fp64(RP.rotate_fp64(x, pos, Dh, base, style), pos + 5, Dh, base, style)
    assert np.allclose(z, RP.rotate_fp64(x, 2 * pos + 5, Dh, base, style), atol=1e-9)


def test_interleaved_equals_half_on_permuted_dims():
    Dh = 32
    x = _rand(4, (3, 2, Dh))
    perm = np.concatenate([np.arange(0, Dh, 2), np.arange(1, Dh, 2)])  # even dims first, then odd
    a = RP.rotate_fp64(x, [3, 50, 9], Dh, 10000.0, "interleaved")
    b = RP.rotate_fp64(x[..., perm], [3, 50, 9], Dh, 10000.0, "half")
    assert np.allclose(a[..., perm], b, atol=1e-13)


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("style", RP.STYLES)
def test_stored_precision_within_rounding_of_the_exact_rotation(dtype, style):
    Dh, base, N, H = 128, 10000.0, 64, 4
    tab = RP.rope_table(4096, Dh, base)
    pos = W.generator(5, W.S_LENGTHS).integers(0, 4096, N)
    raw = W.normal_storage(6, W.S_KNEW, (0,), (N, H, Dh), dtype)
    x = RP.storage_to_f32(raw, dtype).astype(np.float64)
    got = RP.storage_to_f32(RP.apply_rope(raw, pos, tab, style, dtype), dtype).astype(np.float64)
    exact = RP.rotate_fp64(x, pos, Dh, base, style)
    i, j = RP.pair_index(Dh, style)
    mag = np.zeros_like(x)
    mag[..., i] = mag[..., j] = np.abs(x[..., i]) + np.abs(x[..., j])
    ulp = {"bf16": 2.0 ** -8, "fp16": 2.0 ** -11, "fp32": 2.0 ** -24}[dtype]
    bound = ulp * np.abs(exact) + 4 * 2.0 ** -24 * mag + 1e-30
    assert (np.abs(got - exact) <= bound).all()
    if dtype != "fp32":  # nearly every element is the correctly rounded exact value
        assert (RP.to_storage(exact.astype(np.float32), dtype) == RP.apply_rope(raw, pos, tab, style, dtype)).mean() > 0.97


def test_rope_append_scatters_rotated_k_and_raw_v():
    Dh, P, H = 16, 4, 2
    tab = RP.rope_table(64, Dh)
    k_new = W.normal_storage(7, W.S_KNEW, (0,), (3, H, Dh), "bf16")
    v_new = W.normal_storage(7, W.S_VNEW, (0,), (3, H, Dh), "bf16")
    kp = np.zeros((4, H, P, Dh), np.uint16)
    vp = np.zeros_like(kp)
    RP.rope_append(kp, vp, k_new, v_new, [5, -1, 14], [9, 3, 30], tab, "half", "bf16")
    rot = RP.apply_rope(k_new, [9, 3, 30], tab, "half", "bf16")
    assert np.array_equal(kp[1, :, 1], rot[0]) and np.array_equal(vp[1, :, 1], v_new[0])
    assert np.array_equal(kp[3, :, 2], rot[2]) and np.array_equal(vp[3, :, 2], v_new[2])
    assert np.count_nonzero(kp) == np.count_nonzero(rot[0]) + np.count_nonzero(rot[2])


# ---------------------------------------------------------------- planted mistakes
ROPE_MUTANTS = {
    "sign of the sine term": ("out[..., i] = x[..., i] * c - x[..., j] * s", "out[..., i] = x[..., i] * c + x[..., j] * s"),
    "frequency exponent": ("theta = np.power(float(base), -2.0 * k / Dh)", "theta = np.power(float(base), -1.0 * k / Dh)"),
    "half pairing offset": ("return k, k + Dh // 2", "return k, k + Dh // 2 - 1"),
    "stored sum sign": ("(xj * c).astype(np.float32) + (xi * s)", "(xj * c).astype(np.float32) - (xi * s)"),
    "table columns swapped": ("[np.cos(a), np.sin(a)]", "[np.sin(a), np.cos(a)]"),
    "bf16 tie rounding": ("0x7FFF + ((b >> 16) & 1)", "0x8000"),
}


def _pins(mod):
    failed = []
    checks = {
        "worked": lambda: _worked(mod),
        "relative": lambda: _relative(mod),
        "stored": lambda: _stored(mod),
        "ties": lambda: _ties(mod),
    }
    for name, fn in checks.items():
        try:
            fn()
        except AssertionError:
            failed.append(name)
    return failed


def _worked(mod):
    x = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    c1, s1, c01, s01 = 0.5403023058681398, 0.8414709848078965, 0.9950041652780258, 0.09983341664682815
    half = mod.rotate_fp64(x, [1], 4, 100.0, "half")[0, 0]
    assert np.allclose(half, [1 * c1 - 3 * s1, 2 * c01 - 4 * s01, 3 * c1 + 1 * s1, 4 * c01 + 2 * s01], atol=1e-15)
    assert np.array_equal(mod.rope_table(2, 4, 100.0)[1], np.array([c1, c01, s1, s01], np.float32))


def _relative(mod):
    q, k = _rand(1, (1, 1, 64)), _rand(2, (1, 1, 64))
    d = lambda m, n: float((mod.rotate_fp64(q, [m], 64, 1e4, "half") * mod.rotate_fp64(k, [n], 64, 1e4, "half")).sum())
    assert abs(d(103, 100) - d(3, 0)) < 1e-10


def _stored(mod):
    tab = mod.rope_table(512, 64)
    raw = W.normal_storage(6, W.S_KNEW, (0,), (8, 2, 64), "bf16")
    pos = np.arange(8) * 37
    got = mod.storage_to_f32(mod.apply_rope(raw, pos, tab, "half", "bf16"), "bf16").astype(np.float64)
    exact = RP.rotate_fp64(RP.storage_to_f32(raw, "bf16").astype(np.float64), pos, 64, 10000.0, "half")
    assert np.abs(got - exact).max() <= 2.0 ** -8 * np.abs(exact).max() + 1e-6


def _ties(mod):
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], np.float32)  # exact bf16 ties
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mod.f32_to_bf16_bits(x), ref)


def _load_mutant(tmp_path, name, old, new):
    src = open(os.path.join(ROOT, "oracle", "rope.py"), encoding="utf-8").read()
    assert old in src, name
    path = tmp_path / f"rope_mut_{abs(hash(name))}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(path.stem, path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_unmodified_rope_oracle_passes_every_pin():
    assert _pins(RP) == []


@pytest.mark.parametrize("name", sorted(ROPE_MUTANTS))
def test_rope_mutant_is_caught(tmp_path, name):
    old, new = ROPE_MUTANTS[name]
    assert _pins(_load_mutant(tmp_path, name, old, new)), f"mutant '{name}' survived every pin"
