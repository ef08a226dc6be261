"""Parity tolerances of the GPU path against the fp64 oracle.

  bf16 outputs and gradients:  relative L2 <= 1e-2 and max-abs <= 5e-2
  fp32 final state (bf16 path): relative L2 <= 5e-3
  fp32 decode path:             relative L2 <= 1e-5

Reading of the max-abs bound for outputs STORED in bf16: a value of
magnitude m stored in bf16 is off by up to half a bf16 ulp, 2^(floor(log2 m) - 8),
even when computed exactly (0.03125 for m in [8, 16), 0.0625 for m in
[16, 32)).  The bound 5e-2 is applied to the error beyond that storage
rounding: |gpu - oracle| <= 5e-2 + half_ulp_bf16(oracle), elementwise.  The
relative L2 bound is applied as is.  The raw max-abs is returned for reports.
"""
import numpy as np

REL_BF16, ABS_BF16, REL_STATE, REL_F32 = 1e-2, 5e-2, 5e-3, 1e-5


def rel_l2(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


def half_ulp_bf16(ref):
    m = np.abs(np.asarray(ref, np.float64))
    e = np.floor(np.log2(np.maximum(m, 2.0 ** -126)))
    return np.where(m > 0, np.exp2(e - 8), 0.0)


def bf16_errors(x, ref):
    """(rel L2, raw max-abs, max-abs beyond the bf16 storage rounding)."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(x - ref)
    beyond = err - half_ulp_bf16(ref)
    return rel_l2(x, ref), float(err.max(initial=0.0)), float(beyond.max(initial=0.0))


def assert_bf16_close(x, ref, what="output", rel=REL_BF16, abs_=ABS_BF16):
    r, raw, beyond = bf16_errors(x, ref)
    assert r <= rel, "%s: rel L2 %.3g > %.3g" % (what, r, rel)
    assert beyond <= abs_, "%s: max-abs beyond bf16 rounding %.3g > %.3g (raw %.3g)" % (
        what, beyond, abs_, raw)
    return r, raw, beyond
