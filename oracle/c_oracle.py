"""ctypes binding of the C fp64 oracle (``mhc_oracle.c``). TEST INFRASTRUCTURE ONLY.

Array conventions: bf16 tensors are passed as ``numpy.uint16`` bit patterns; fp32 inputs as
``numpy.float32``; every result is ``numpy.float64``. Shapes follow ``mhc_oracle.h``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mhc_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_F = ctypes.POINTER(ctypes.c_float)
_U16 = ctypes.POINTER(ctypes.c_uint16)
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (-O2 -fopenmp, IEEE arithmetic, no fast-math)."""
    stale = not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "mhc_oracle.h"))
    )
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", "-o", tmp, _SRC, "-lm"],
            check=True,
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    lib.mhc_oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.mhc_oracle_bf16_to_double.restype = ctypes.c_double
    lib.mhc_oracle_round_bf16.argtypes = [_D, _I64, _D]
    lib.mhc_oracle_norm_project.argtypes = [_U16, _F, _I64, _I64, ctypes.c_double, _D, _D, _D]
    lib.mhc_oracle_sinkhorn.argtypes = [_D, _I64, ctypes.c_int, ctypes.c_double, _D]
    lib.mhc_oracle_sinkhorn_converge.argtypes = [_D, _I64, ctypes.c_double, ctypes.c_double,
                                                 ctypes.c_int, _D]
    lib.mhc_oracle_sinkhorn_converge.restype = ctypes.c_int
    lib.mhc_oracle_sinkhorn_variant.argtypes = [_D, _I64, ctypes.c_int, ctypes.c_double,
                                                ctypes.c_int, _D]
    lib.mhc_oracle_coefficients.argtypes = [_D, _D, _F, _F, _I64, ctypes.c_double,
                                            ctypes.c_double, ctypes.c_int, ctypes.c_double,
                                            _D, _D, _D, _D]
    lib.mhc_oracle_aggregate.argtypes = [_U16, _D, _I64, _I64, _D]
    lib.mhc_oracle_pre.argtypes = [_U16, _F, _F, _F, _I64, _I64, ctypes.c_double,
                                   ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                   ctypes.c_double, _D, _D, _D, _D, _D, _D]
    lib.mhc_oracle_post.argtypes = [_U16, _U16, _F, _F, _I64, _I64, _D]
    lib.mhc_oracle_threads.restype = ctypes.c_int
    lib.mhc_oracle_set_threads.argtypes = [ctypes.c_int]
    _lib = lib
    return lib


def _c(a, dtype, ptr):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ptr)


def threads() -> int:
    return int(_load().mhc_oracle_threads())


def set_threads(n: int) -> None:
    """OpenMP threads for later oracle calls (the CPU baseline times 1 thread and all of them)."""
    _load().mhc_oracle_set_threads(int(n))


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns (vectorised in NumPy: a shift into the fp32 high half)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(v) -> np.ndarray:
    """Round fp64 values to bf16 (RNE); returns float64 holding the exact bf16 values."""
    v, pv = _c(v, np.float64, _D)
    out = np.empty_like(v)
    _load().mhc_oracle_round_bf16(pv, v.size, out.ctypes.data_as(_D))
    return out


def norm_project(R, hc_fn, rms_eps=1e-6):
    """Steps a1-a2. R: uint16 [T,4,H]; hc_fn: float32 [4H,24]. Returns (ss, rstd, raw[T,24])."""
    T, hc, H = R.shape
    assert hc == 4 and hc_fn.shape == (4 * H, 24)
    R, pR = _c(R, np.uint16, _U16)
    W, pW = _c(hc_fn, np.float32, _F)
    ss = np.empty(T)
    rstd = np.empty(T)
    raw = np.empty((T, 24))
    _load().mhc_oracle_norm_project(pR, pW, T, H, rms_eps, ss.ctypes.data_as(_D),
                                    rstd.ctypes.data_as(_D), raw.ctypes.data_as(_D))
    return ss, rstd, raw


def sinkhorn(logits, iters=20, eps=1e-6):
    """Step a4/a7 on logits [T,4,4] (or [T,16]); returns comb [T,4,4] ([old][new]): softmax of
    each row plus eps, then `iters` (row, column) normalisation rounds."""
    lg, pl = _c(logits, np.float64, _D)
    T = lg.size // 16
    out = np.empty((T, 4, 4))
    _load().mhc_oracle_sinkhorn(pl, T, int(iters), float(eps), out.ctypes.data_as(_D))
    return out


def sinkhorn_converge(logits, eps=1e-6, tol=1e-12, max_iters=10000):
    lg, pl = _c(logits, np.float64, _D)
    T = lg.size // 16
    out = np.empty((T, 4, 4))
    used = _load().mhc_oracle_sinkhorn_converge(pl, T, float(eps), float(tol), int(max_iters),
                                                out.ctypes.data_as(_D))
    return out, used


def sinkhorn_variant(logits, iters=20, eps=1e-6, variant=1):
    """Another reading of the Sinkhorn step, for the reading-gap report only (see mhc_oracle.h):
    variant 1 = eps in the row/column sums, none on the entries; variant 2 = an extra column
    normalisation straight after the softmax."""
    lg, pl = _c(logits, np.float64, _D)
    T = lg.size // 16
    out = np.empty((T, 4, 4))
    _load().mhc_oracle_sinkhorn_variant(pl, T, int(iters), float(eps), int(variant),
                                        out.ctypes.data_as(_D))
    return out


def coefficients(raw, rstd, scale, base, pre_eps=0.0, post_mult=2.0, iters=20, eps=1e-6):
    """Steps a3-a4. Returns (logits[T,24], pre[T,4], post[T,4], comb[T,4,4])."""
    raw, praw = _c(raw, np.float64, _D)
    rstd, prstd = _c(rstd, np.float64, _D)
    sc, psc = _c(scale, np.float32, _F)
    bs, pbs = _c(base, np.float32, _F)
    T = rstd.size
    logits = np.empty((T, 24))
    pre_ = np.empty((T, 4))
    post_ = np.empty((T, 4))
    comb = np.empty((T, 4, 4))
    _load().mhc_oracle_coefficients(praw, prstd, psc, pbs, T, pre_eps, post_mult, int(iters), eps,
                                    logits.ctypes.data_as(_D), pre_.ctypes.data_as(_D),
                                    post_.ctypes.data_as(_D), comb.ctypes.data_as(_D))
    return logits, pre_, post_, comb


def aggregate(R, pre_coef):
    """Step a5 with the given (fp64) pre coefficients. Returns y [T,H] in fp64."""
    T, hc, H = R.shape
    R, pR = _c(R, np.uint16, _U16)
    p, pp = _c(pre_coef, np.float64, _D)
    y = np.empty((T, H))
    _load().mhc_oracle_aggregate(pR, pp, T, H, y.ctypes.data_as(_D))
    return y


def pre(R, hc_fn, scale, base, rms_eps=1e-6, pre_eps=0.0, post_mult=2.0, iters=20, eps=1e-6,
        want_y=True):
    """Whole pre-map (a1-a5). Returns dict of fp64 arrays: rstd, logits, pre, post, comb, y."""
    T, hc, H = R.shape
    R, pR = _c(R, np.uint16, _U16)
    W, pW = _c(hc_fn, np.float32, _F)
    sc, psc = _c(scale, np.float32, _F)
    bs, pbs = _c(base, np.float32, _F)
    out = {
        "rstd": np.empty(T), "logits": np.empty((T, 24)), "pre": np.empty((T, 4)),
        "post": np.empty((T, 4)), "comb": np.empty((T, 4, 4)),
    }
    y = np.empty((T, H)) if want_y else None
    _load().mhc_oracle_pre(pR, pW, psc, pbs, T, H, rms_eps, pre_eps, post_mult, int(iters), eps,
                           out["rstd"].ctypes.data_as(_D), out["logits"].ctypes.data_as(_D),
                           out["pre"].ctypes.data_as(_D), out["post"].ctypes.data_as(_D),
                           out["comb"].ctypes.data_as(_D),
                           y.ctypes.data_as(_D) if want_y else None)
    out["y"] = y
    return out


def post(x, R, post_coef, comb):
    """Step a6 with fp32 post [T,4] and comb [T,4,4]. Returns out [T,4,H] in fp64."""
    T, hc, H = R.shape
    x, px = _c(x, np.uint16, _U16)
    R, pR = _c(R, np.uint16, _U16)
    p, pp = _c(post_coef, np.float32, _F)
    c, pc = _c(comb, np.float32, _F)
    assert p.size == T * 4 and c.size == T * 16 and x.size == T * H
    out = np.empty((T, 4, H))
    _load().mhc_oracle_post(px, pR, pp, pc, T, H, out.ctypes.data_as(_D))
    return out
