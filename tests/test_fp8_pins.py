"""Pins of the FP8 (E4M3) K/V oracle (oracle/fp8.py): the format against
torch's float8_e4m3fn and closed forms, the quantiser's error bound, the fp8
decode against brute force; planted mistakes must fail a pin."""
import importlib.util
import math
import os

import numpy as np
import pytest
import torch

from helpers import ROOT
from oracle import fp8 as F
from oracle import reference as R
from paged_kv_cache_433_b200 import workloads as W


def test_code_values_match_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = F.E4M3_TABLE
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine)) and nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ref[~nan], mine[~nan])


def test_encoder_matches_torch_cast_in_range_including_ties():
    g = W.generator(50, W.S_K)
    x = np.concatenate([g.standard_normal(20000) * 40, g.standard_normal(5000) * 0.01])
    finite = F.E4M3_TABLE[np.isfinite(F.E4M3_TABLE)]
    pos = np.unique(finite[finite >= 0])
    mids = (pos[:-1] + pos[1:]) / 2  # exact ties between neighbouring codes
    x = np.concatenate([x, mids, -mids])
    x = np.clip(x, -448, 448).astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_encode(x), ref)


@pytest.mark.parametrize("x,code", [
    (448.0, 0x7E), (1000.0, 0x7E), (-1000.0, 0xFE), (464.0, 0x7E), (1.0, 0x38), (-2.0, 0xC0),
    (2.0 ** -9, 0x01), (2.0 ** -10, 0x00), (3 * 2.0 ** -10, 0x02), (1.0625, 0x38), (1.1875, 0x3A),
    (-0.0, 0x80), (0.0, 0x00), (float("nan"), 0x7F), (240.0, 0x77),
])
def test_encoder_closed_forms(x, code):
    assert int(F.e4m3_encode(np.array([x]))[0]) == code


def test_quantiser_relative_error_bound_and_division():
    raw = W.normal_storage(52, W.S_KNEW, (0,), (64, 4, 32), "bf16")
    scale = np.array([0.01, 0.02, 0.005, 0.03], np.float32)
    codes = F.quantize(raw, "bf16", scale)
    x = R.decode_storage(raw, "bf16")
    y = (x.astype(np.float32) / scale[None, :, None]).astype(np.float64)  # the quantiser's input
    dq = F.e4m3_decode(codes)
    normal = (np.abs(y) >= 2.0 ** -6) & (np.abs(y) <= 448)
    assert (np.abs(dq - y)[normal] <= 2.0 ** -4 * np.abs(y)[normal]).all()
    sub = np.abs(y) < 2.0 ** -6
    assert (np.abs(dq - y)[sub] <= 2.0 ** -10 + 1e-18).all()
    assert (dq[np.abs(y) > 448] == np.sign(y[np.abs(y) > 448]) * 448).all()


def _brute(q, q_dtype, kc, vc, ks, vs, tab, lens, scale):
    """Per (b, h): materialise the read K / V rows with Python floats and take the softmax."""
    B, H_q, Dh = q.shape
    H_kv, P = kc.shape[1], kc.shape[2]
    g = H_q // H_kv
    qd = R.decode_storage(q, q_dtype)
    out = np.zeros((B, H_q, Dh))
    for b in range(B):
        for h in range(H_q):
            kvh = h // g
            s, rows = [], []
            for t in range(int(lens[b])):
                page, off = int(tab[b][t // P]), t % P
                k = [F.e4m3_value(int(c)) * float(np.float32(ks[kvh])) for c in kc[page, kvh, off]]
                v = [F.e4m3_value(int(c)) * float(np.float32(vs[kvh])) for c in vc[page, kvh, off]]
                s.append(scale * sum(qd[b, h, d] * k[d] for d in range(Dh)))
                rows.append(v)
            m = max(s)
            w = [math.exp(x - m) for x in s]
            tot = sum(w)
            out[b, h] = [sum(w[i] * rows[i][d] for i in range(len(w))) / tot for d in range(Dh)]
    return out


def _tiny():
    B, H_q, H_kv, Dh, P = 2, 4, 2, 8, 4
    g = W.generator(53, W.S_K)
    kc = g.integers(0, 256, (5, H_kv, P, Dh)).astype(np.uint8)
    vc = g.integers(0, 256, (5, H_kv, P, Dh)).astype(np.uint8)
    kc[(kc & 0x7F) == 0x7F] = 0x10  # no NaN codes
    vc[(vc & 0x7F) == 0x7F] = 0x22
    q = W.normal_storage(53, W.S_Q, (0,), (B, H_q, Dh), "fp16")
    tab = np.array([[3, 0], [4, 1]], np.int32)
    lens = np.array([7, 3], np.int32)
    ks = np.array([0.0125, 0.003], np.float32)
    vs = np.array([0.25, 0.07], np.float32)
    return q, kc, vc, ks, vs, tab, lens, 1 / math.sqrt(Dh)


def test_fp8_decode_matches_brute_force():
    q, kc, vc, ks, vs, tab, lens, scale = _tiny()
    got = F.paged_decode_fp8(q, "fp16", kc, vc, ks, vs, tab, lens, scale)
    ref = _brute(q, "fp16", kc, vc, ks, vs, tab, lens, scale)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_append_fp8_writes_quantised_codes():
    P, H, Dh = 4, 2, 16
    kp = np.zeros((3, H, P, Dh), np.uint8)
    vp = np.zeros_like(kp)
    kn = W.normal_storage(54, W.S_KNEW, (0,), (2, H, Dh), "fp16")
    vn = W.normal_storage(54, W.S_VNEW, (0,), (2, H, Dh), "fp16")
    ks, vs = np.array([0.01, 0.02], np.float32), np.array([0.03, 0.04], np.float32)
    F.append_fp8(kp, vp, kn, vn, "fp16", ks, vs, [6, -1])
    assert np.array_equal(kp[1, :, 2], F.quantize(kn, "fp16", ks)[0])
    assert np.array_equal(vp[1, :, 2], F.quantize(vn, "fp16", vs)[0])
    assert np.count_nonzero(kp[0]) == 0 and np.count_nonzero(kp[2]) == 0


# ---------------------------------------------------------------- planted mistakes
FP8_MUTANTS = {
    "subnormal exponent": ("return s * m * 2.0 ** -9", "return s * m * 2.0 ** -10"),
    "exponent bias": ("2.0 ** (e - 7)", "2.0 ** (e - 8)"),
    "ties to odd": ("((d_hi == d_lo) & (hi % 2 == 0))", "((d_hi == d_lo) & (hi % 2 == 1))"),
    "overflow to NaN": ("code = np.where(a >= E4M3_MAX, np.uint8(0x7E), code)",
                        "code = np.where(a > E4M3_MAX, np.uint8(0x7F), code)"),
    "v scale dropped": ("* vs[h]", "* 1.0"),
    "k scale dropped": ("float(scale) * ks[h]", "float(scale)"),
    "multiply by the scale": ("e4m3_encode((x / s).astype(np.float32))", "e4m3_encode((x * s).astype(np.float32))"),
}


def _load_mutant(tmp_path, name, old, new):
    src = open(os.path.join(ROOT, "oracle", "fp8.py"), encoding="utf-8").read()
    assert old in src, name
    pkg = tmp_path / "oracle_mut"
    pkg.mkdir()
    path = pkg / "fp8_mut.py"
    path.write_text(src.replace(old, new).replace("from . import reference as R", "from oracle import reference as R"))
    spec = importlib.util.spec_from_file_location("fp8_mut_" + str(abs(hash(name))), path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _pins(mod):
    failed = []
    for name, fn in [("table", lambda: _pin_table(mod)), ("closed", lambda: _pin_closed(mod)),
                     ("quant", lambda: _pin_quant(mod)), ("brute", lambda: _pin_brute(mod))]:
        try:
            fn()
        except AssertionError:
            failed.append(name)
    return failed


def _pin_table(mod):
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], mod.E4M3_TABLE[ok])


def _pin_closed(mod):
    for x, code in [(1000.0, 0x7E), (3 * 2.0 ** -10, 0x02), (1.0625, 0x38), (2.0 ** -9, 0x01)]:
        assert int(mod.e4m3_encode(np.array([x]))[0]) == code


def _pin_quant(mod):
    raw = W.normal_storage(52, W.S_KNEW, (0,), (16, 2, 32), "bf16")
    scale = np.array([0.01, 0.02], np.float32)
    y = (R.decode_storage(raw, "bf16").astype(np.float32) / scale[None, :, None]).astype(np.float64)
    dq = F.e4m3_decode(mod.quantize(raw, "bf16", scale))
    normal = (np.abs(y) >= 2.0 ** -6) & (np.abs(y) <= 448)
    assert (np.abs(dq - y)[normal] <= 2.0 ** -4 * np.abs(y)[normal]).all()


def _pin_brute(mod):
    q, kc, vc, ks, vs, tab, lens, scale = _tiny()
    got = mod.paged_decode_fp8(q, "fp16", kc, vc, ks, vs, tab, lens, scale)
    assert np.allclose(got, _brute(q, "fp16", kc, vc, ks, vs, tab, lens, scale), rtol=1e-12, atol=1e-12)


def test_unmodified_fp8_oracle_passes_every_pin():
    assert _pins(F) == []


@pytest.mark.parametrize("name", sorted(FP8_MUTANTS))
def test_fp8_mutant_is_caught(tmp_path, name):
    old, new = FP8_MUTANTS[name]
    assert _pins(_load_mutant(tmp_path, name, old, new)), f"mutant '{name}' survived every pin"
