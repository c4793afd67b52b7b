"""Shared test helpers (no method arithmetic: fixtures, paths, tolerances)."""
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")

# Attention tolerance against the fp64 oracle: |gpu - ref| <= ATOL + RTOL * |ref|.
# bf16/fp16 K/V: 2e-3 / 2e-3 (the contract). fp32 K/V: 1e-5 / 1e-5 (tighter,
# from fp32 accumulation over <= a few thousand terms of magnitude ~1).
TOL = {"bf16": (2e-3, 2e-3), "fp16": (2e-3, 2e-3), "fp32": (1e-5, 1e-5)}


def golden(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        return json.load(f)
