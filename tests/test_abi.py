"""The C ABI on the host (no GPU needed): libmhc.so loads, exports every entry point include/mhc.h
declares, and rejects bad arguments before any CUDA call. The pointers below are fake addresses;
every case returns during host-side validation, before the library binds a device or launches."""

import ctypes
import os
import re
import subprocess

import pytest

import mhc_hyper_connection_02_b200 as mhc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mhc.h")


@pytest.fixture(scope="module")
def L():
    from mhc_hyper_connection_02_b200 import build
    build.build()
    return mhc.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MHC_API\s+[\w\s\*]+?\b(mhc_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("mhc_pre", "mhc_post", "mhc_sinkhorn", "mhc_pre_workspace_bytes",
                 "mhc_status_string"):
        assert name in syms
    assert set(syms) == set(mhc.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", mhc.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(mhc_\w+)$", out, re.M))
    assert set(declared_symbols()) <= exported
    for name in declared_symbols():
        assert hasattr(L, name)
    # nothing else leaks out of the library (kernels and helpers are hidden)
    assert not any(s.startswith("_ZN3mhc") for s in re.findall(r"\bT\s+(\S+)$", out, re.M))


def test_build_targets_sm100a_only():
    from mhc_hyper_connection_02_b200 import build
    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1 and "fast-math" not in flags


def test_constants_and_defaults(L):
    assert mhc.status_string(0) == "MHC_OK"
    assert mhc.status_string(mhc.MHC_ERR_ALIAS) == "MHC_ERR_ALIAS"
    assert mhc.status_string(-99) == "MHC_ERR_UNKNOWN"
    assert L.mhc_version() >= 100
    p = mhc.default_params()
    assert p.sinkhorn_iters == 20 and abs(p.sinkhorn_eps - 1e-6) < 1e-12
    assert abs(p.rms_eps - 1e-6) < 1e-12 and p.pre_eps == 0.0 and p.post_mult == 2.0


def test_workspace_bytes(L):
    assert mhc.workspace_bytes(0, 512) == 0 and mhc.workspace_bytes(64, 0) == 0
    for T, H in ((1, 7168), (32, 7168), (64, 512), (3000, 1000), (8192, 7168), (5, 127)):
        n = mhc.workspace_bytes(T, H)
        assert n > 0 and n % 256 == 0
        assert n < 64 * 2 ** 20 or T * H > 2 ** 24


# fake, well-separated device addresses (never dereferenced: validation fails first)
A = 1 << 40
R_, X_, P_, C_, O_ = A, A + (1 << 34), A + (2 << 34), A + (3 << 34), A + (4 << 34)


def post_call(L, x=X_, R=R_, post=P_, comb=C_, out=O_, T=8, H=64, path=0):
    return L.mhc_post_with_path(x, R, post, comb, out, T, H, path, None)


def test_post_validation(L):
    assert post_call(L, T=0) == mhc.MHC_OK                       # empty: no launch
    assert post_call(L, T=-1) == mhc.MHC_ERR_INVALID_ARG
    assert post_call(L, H=0) == mhc.MHC_ERR_INVALID_ARG
    assert post_call(L, x=None) == mhc.MHC_ERR_INVALID_ARG
    assert post_call(L, out=None) == mhc.MHC_ERR_INVALID_ARG
    assert post_call(L, out=R_ + 2) == mhc.MHC_ERR_ALIAS         # partial overlap with R
    assert post_call(L, out=X_ - 16) == mhc.MHC_ERR_ALIAS        # overlaps x
    assert post_call(L, path=99) == mhc.MHC_ERR_INVALID_ARG
    assert post_call(L, H=127, path=mhc.POST_PATH_VEC8) == mhc.MHC_ERR_UNSUPPORTED
    assert post_call(L, R=R_ + 2, out=O_, path=mhc.POST_PATH_PERSISTENT) == mhc.MHC_ERR_UNSUPPORTED
    assert post_call(L, T=2 ** 62) == mhc.MHC_ERR_INVALID_ARG    # size overflow


def test_sinkhorn_validation(L):
    f = L.mhc_sinkhorn
    assert f(A, A + (1 << 30), 0, 0, 20, ctypes.c_float(1e-6), None) == mhc.MHC_OK
    assert f(A, A + (1 << 30), -1, 0, 20, ctypes.c_float(1e-6), None) == mhc.MHC_ERR_INVALID_ARG
    assert f(A, A + (1 << 30), 4, 0, 0, ctypes.c_float(1e-6), None) == mhc.MHC_ERR_INVALID_ARG
    assert f(A, A + (1 << 30), 4, 0, 20, ctypes.c_float(0.0), None) == mhc.MHC_ERR_INVALID_ARG
    assert f(A, A + (1 << 30), 4, 0, 20, ctypes.c_float(float("nan")), None) == mhc.MHC_ERR_INVALID_ARG
    assert f(None, A, 4, 0, 20, ctypes.c_float(1e-6), None) == mhc.MHC_ERR_INVALID_ARG
    assert f(A, A + 4, 4, 0, 20, ctypes.c_float(1e-6), None) == mhc.MHC_ERR_ALIAS


def pre_call(L, T=16, H=64, ws=None, wsb=None, params=None, path=0, **over):
    ptr = dict(R=A, W=A + (1 << 34), S=A + (2 << 34), B=A + (3 << 34), y=A + (4 << 34),
               pre=A + (5 << 34), post=A + (6 << 34), comb=A + (7 << 34))
    ptr.update(over)
    need = mhc.workspace_bytes(T, H)
    ws = A + (8 << 34) if ws is None else ws
    wsb = need if wsb is None else wsb
    p = ctypes.byref(params) if params is not None else None
    return L.mhc_pre_with_path(ptr["R"], ptr["W"], ptr["S"], ptr["B"], ptr["y"], ptr["pre"],
                               ptr["post"], ptr["comb"], ws, wsb, T, H, p, path, None)


def test_pre_validation(L):
    assert pre_call(L, T=0) == mhc.MHC_OK
    assert pre_call(L, T=-3) == mhc.MHC_ERR_INVALID_ARG
    assert pre_call(L, H=-1) == mhc.MHC_ERR_INVALID_ARG
    assert pre_call(L, R=None) == mhc.MHC_ERR_INVALID_ARG
    assert pre_call(L, comb=None) == mhc.MHC_ERR_INVALID_ARG
    assert pre_call(L, wsb=mhc.workspace_bytes(16, 64) - 1) == mhc.MHC_ERR_WORKSPACE_TOO_SMALL
    assert pre_call(L, ws=0) == mhc.MHC_ERR_WORKSPACE_TOO_SMALL
    assert pre_call(L, y=A + 8) == mhc.MHC_ERR_ALIAS               # y overlaps R
    assert pre_call(L, post=A + (5 << 34) + 4) == mhc.MHC_ERR_ALIAS  # post overlaps pre
    assert pre_call(L, path=7) == mhc.MHC_ERR_INVALID_ARG
    for field, bad in (("sinkhorn_iters", 0), ("sinkhorn_eps", 0.0), ("rms_eps", -1.0),
                       ("pre_eps", -1e-3), ("post_mult", float("inf")),
                       ("sinkhorn_eps", float("nan"))):
        p = mhc.default_params()
        setattr(p, field, bad)
        assert pre_call(L, params=p) == mhc.MHC_ERR_INVALID_ARG, field


def test_python_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(mhc, "_lib", None)
    monkeypatch.setattr(mhc, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        mhc.lib()
