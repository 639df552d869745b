"""Comparison rules for GPU results against the fp64 oracle (test helper, no method arithmetic).

Coefficients (pre, post, comb, fp32): max |gpu - oracle| <= 1e-5.

bf16 outputs (y, out): the stated rule is |gpu - bf16(v)| <= max(ulp_bf16(bf16(v)), 2e-2 * |v|),
v the fp64 oracle value. Where the result cancels (|v| much smaller than its terms) fp32 evaluation
cannot meet that rule in principle, so an element also passes under the bound derived from the
arithmetic:  ulp_bf16(bf16(v)) + E, with E the fp32 evaluation error of the kernel's own expression
(n_ops roundings of at most 2^-24 relative to the running sum of |terms|) plus, for y, the error the
admitted coefficient difference (<= 1e-5 per gate) carries in. Tests report how many elements needed
the derived bound; a wrong term, index or sign produces errors of the size of the terms themselves
and fails both rules.
"""

import numpy as np

COEF_TOL = 1e-5
REL = 2e-2
U32 = 2.0 ** -24


def bf16_bits_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(
        np.float64)


def ulp_bf16(v):
    """Spacing of bf16 numbers at |v| (v already a bf16 value); the subnormal spacing at 0."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.where(a > 0, np.maximum(e, -126.0), -126.0)
    return np.ldexp(1.0, (e - 7).astype(np.int64))


def check_bf16(gpu_bits, v, v_bf16, extra_bound):
    """Returns (n_fail, n_needed_derived, worst_ratio). extra_bound is the derived term E."""
    g = bf16_bits_to_f64(gpu_bits)
    err = np.abs(g - v_bf16)
    u = ulp_bf16(v_bf16)
    strict = np.maximum(u, REL * np.abs(v))
    derived = u + extra_bound
    tol = np.maximum(strict, derived)
    fail = err > tol
    need = (err > strict) & ~fail
    ratio = float(np.max(err / tol)) if err.size else 0.0
    return int(fail.sum()), int(need.sum()), ratio


def check_coef(gpu, ref, name):
    d = float(np.max(np.abs(np.asarray(gpu, np.float64) - ref))) if np.size(ref) else 0.0
    assert d <= COEF_TOL, f"{name}: max |gpu - oracle| = {d:.3e} > {COEF_TOL}"
    return d
