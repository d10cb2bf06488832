"""Shared test helpers: tolerance checks and lazy builds (no layer arithmetic here)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# The layer's floating-point tolerance: max |gpu - ref| <= 2e-2 * max |ref| and
# sum |gpu - ref| / sum |ref| <= 5e-3 (a mean relative error that stays finite near 0).
TOL_MAX = 2e-2
TOL_MEAN = 5e-3


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def close_report(got_bits, ref_bits):
    got, ref = bf16_bits_to_f64(got_bits), bf16_bits_to_f64(ref_bits)
    err = np.abs(got - ref)
    scale = np.abs(ref).max()
    return {
        "max_err": float(err.max()) if err.size else 0.0,
        "max_ref": float(scale) if err.size else 0.0,
        "mean_rel": float(err.sum() / max(np.abs(ref).sum(), 1e-30)),
        "finite": bool(np.isfinite(got).all()),
    }


def assert_layer_close(got_bits, ref_bits, tol_max=TOL_MAX, tol_mean=TOL_MEAN):
    r = close_report(got_bits, ref_bits)
    assert r["finite"], r
    if r["max_ref"] == 0:
        assert r["max_err"] == 0, r
        return r
    assert r["max_err"] <= tol_max * r["max_ref"], r
    assert r["mean_rel"] <= tol_mean, r
    return r


def header_symbols():
    """Names of every function declared in include/*.h."""
    names = []
    inc = os.path.join(ROOT, "include")
    for fn in sorted(os.listdir(inc)):
        if fn.endswith(".h"):
            text = open(os.path.join(inc, fn)).read()
            names += re.findall(r"CHORD_API[^;(]*?\b(chord_\w+)\s*\(", text)
    return names


def ensure_built():
    """Build libchord.so and the oracle if missing (nvcc/gcc; no GPU needed)."""
    from w4a16_int4_mixture_align_b200 import build as b
    import oracle
    b.build()
    oracle.build()
