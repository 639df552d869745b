"""mHC (manifold-constrained hyper-connection, HC = 4) pre-map / post-map on B200.

Thin Python binding of the ``libmhc.so`` C ABI (``include/mhc.h``): argument marshalling only.
PyTorch provides device memory and streams; every step of the path runs in the library's CUDA
kernels. There is no CPU fallback: if ``libmhc.so`` has not been built, every call raises.

    import torch, mhc_hyper_connection_02_b200 as mhc
    y, pre, post, comb = mhc.pre(R, hc_fn, hc_scale, hc_base)      # R [T,4,H] bf16 on cuda
    out = mhc.post(x, R, post, comb)                               # out [T,4,H] bf16
"""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmhc.so")

# Status codes and path selectors (mirrors include/mhc.h).
MHC_OK = 0
MHC_ERR_INVALID_ARG = -1
MHC_ERR_WORKSPACE_TOO_SMALL = -2
MHC_ERR_ALIAS = -3
MHC_ERR_CUDA = -4
MHC_ERR_UNSUPPORTED = -5
MHC_ERR_TIMEOUT = -6
MHC_ERR_SCRATCH_LIMIT = -7
NOALLOC_SCRATCH_BYTES = 4 << 20

PATH_AUTO = 0
PRE_PATH_CUDA_CORE = 1
PRE_PATH_TENSOR = 2
PRE_PATH_TENSOR_SPLIT = 3
PRE_PATH_TENSOR_FUSED = 4
PRE_PATH_TENSOR_WAVE = 5
POST_PATH_VEC8 = 11
POST_PATH_PERSISTENT = 12
POST_PATH_SCALAR = 13

EXPORTED_SYMBOLS = (
    "mhc_default_params", "mhc_pre", "mhc_pre_workspace_bytes", "mhc_post", "mhc_sinkhorn",
    "mhc_pre_with_path", "mhc_post_with_path", "mhc_device_status", "mhc_status_string",
    "mhc_version", "mhc_launch_count", "mhc_pre_noalloc", "mhc_pre_big_fuse",
    "mhc_pre_big_fuse_with_prenorm", "mhc_expand", "mhc_head_mean", "mhc_head",
    "mhc_head_workspace_bytes", "mhc_post_project", "mhc_post_project_splits",
    "mhc_post_project_workspace_bytes", "mhc_post_backward", "mhc_pre_backward",
    "mhc_pre_backward_workspace_bytes", "mhc_selftest_wait_timeout",
)


class MhcError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what} failed: {status_string(status)} ({status})")


class Params(ctypes.Structure):
    _fields_ = [("sinkhorn_iters", ctypes.c_int), ("sinkhorn_eps", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("pre_eps", ctypes.c_float),
                ("post_mult", ctypes.c_float)]


_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def lib() -> ctypes.CDLL:
    """The loaded ``libmhc.so`` with argument types set. Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libmhc.so is not built ({LIB_PATH}); run `python -m mhc_hyper_connection_02_b200.build`."
            " There is no CPU fallback.")
    L = ctypes.CDLL(LIB_PATH)
    L.mhc_default_params.restype = Params
    L.mhc_default_params.argtypes = []
    L.mhc_pre.restype = ctypes.c_int
    L.mhc_pre.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I64, _I64,
                          ctypes.POINTER(Params), _P]
    L.mhc_pre_with_path.restype = ctypes.c_int
    L.mhc_pre_with_path.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I64,
                                    _I64, ctypes.POINTER(Params), ctypes.c_int, _P]
    L.mhc_pre_workspace_bytes.restype = ctypes.c_size_t
    L.mhc_pre_workspace_bytes.argtypes = [_I64, _I64]
    L.mhc_post.restype = ctypes.c_int
    L.mhc_post.argtypes = [_P, _P, _P, _P, _P, _I64, _I64, _P]
    L.mhc_post_with_path.restype = ctypes.c_int
    L.mhc_post_with_path.argtypes = [_P, _P, _P, _P, _P, _I64, _I64, ctypes.c_int, _P]
    L.mhc_sinkhorn.restype = ctypes.c_int
    L.mhc_sinkhorn.argtypes = [_P, _P, _I64, _I64, ctypes.c_int, ctypes.c_float, _P]
    L.mhc_device_status.restype = ctypes.c_int
    L.mhc_device_status.argtypes = [_P]
    L.mhc_selftest_wait_timeout.restype = ctypes.c_int
    L.mhc_selftest_wait_timeout.argtypes = [_I64, _P]
    L.mhc_status_string.restype = ctypes.c_char_p
    L.mhc_status_string.argtypes = [ctypes.c_int]
    L.mhc_version.restype = ctypes.c_int
    L.mhc_version.argtypes = []
    L.mhc_pre_noalloc.restype = ctypes.c_int
    L.mhc_pre_noalloc.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64,
                                  ctypes.POINTER(Params), _P]
    L.mhc_pre_big_fuse.restype = ctypes.c_int
    L.mhc_pre_big_fuse.argtypes = [_P, _P, ctypes.c_int, _I64, _P, _P, _P, _P, _P, _P, _P, _I64,
                                   _I64, ctypes.POINTER(Params), _P]
    L.mhc_pre_big_fuse_with_prenorm.restype = ctypes.c_int
    L.mhc_pre_big_fuse_with_prenorm.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64,
                                                ctypes.POINTER(Params), _P]
    L.mhc_expand.restype = ctypes.c_int
    L.mhc_expand.argtypes = [_P, _P, _I64, _I64, _P]
    L.mhc_head_mean.restype = ctypes.c_int
    L.mhc_head_mean.argtypes = [_P, _P, _I64, _I64, _P]
    L.mhc_head_workspace_bytes.restype = ctypes.c_size_t
    L.mhc_head_workspace_bytes.argtypes = [_I64, _I64]
    L.mhc_head.restype = ctypes.c_int
    L.mhc_head.argtypes = [_P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I64, _I64,
                           ctypes.c_float, ctypes.c_float, _P]
    L.mhc_post_project_splits.restype = ctypes.c_int
    L.mhc_post_project_splits.argtypes = [_I64, _I64]
    L.mhc_post_project_workspace_bytes.restype = ctypes.c_size_t
    L.mhc_post_project_workspace_bytes.argtypes = [_I64, _I64]
    L.mhc_post_project.restype = ctypes.c_int
    L.mhc_post_project.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I64,
                                   _I64, _P]
    L.mhc_post_backward.restype = ctypes.c_int
    L.mhc_post_backward.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _P]
    L.mhc_pre_backward_workspace_bytes.restype = ctypes.c_size_t
    L.mhc_pre_backward_workspace_bytes.argtypes = [_I64, _I64]
    L.mhc_pre_backward.restype = ctypes.c_int
    L.mhc_pre_backward.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                   ctypes.c_size_t, _I64, _I64, ctypes.POINTER(Params), _P]
    L.mhc_launch_count.restype = ctypes.c_uint64
    L.mhc_launch_count.argtypes = []
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().mhc_status_string(int(status)).decode()


def default_params() -> Params:
    return lib().mhc_default_params()


def make_params(iters=None, eps=None, rms_eps=None, pre_eps=None, post_mult=None) -> Params:
    p = default_params()
    if iters is not None:
        p.sinkhorn_iters = int(iters)
    if eps is not None:
        p.sinkhorn_eps = float(eps)
    if rms_eps is not None:
        p.rms_eps = float(rms_eps)
    if pre_eps is not None:
        p.pre_eps = float(pre_eps)
    if post_mult is not None:
        p.post_mult = float(post_mult)
    return p


def workspace_bytes(T: int, H: int) -> int:
    return int(lib().mhc_pre_workspace_bytes(int(T), int(H)))


def _check(st: int, what: str) -> None:
    if st != MHC_OK:
        raise MhcError(st, what)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(getattr(stream, "cuda_stream", stream)))


def _need(t, dtype, shape, name):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor "
                         f"(got {t.dtype}, cuda={t.is_cuda}, contiguous={t.is_contiguous()})")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} shape {tuple(t.shape)} != {tuple(shape)}")


def pre(R, hc_fn, hc_scale, hc_base, *, y=None, pre=None, post=None, comb=None, workspace=None,
        params: Params | None = None, path: int = PATH_AUTO, stream=None):
    """Fused pre-map. R [T,4,H] bf16; hc_fn [4H,24], hc_scale [3], hc_base [24] fp32.
    Returns (y [T,H] bf16, pre [T,4], post [T,4], comb [T,4,4] fp32)."""
    import torch
    _need(R, torch.bfloat16, None, "R")
    T, hc, H = R.shape
    if hc != 4:
        raise ValueError("R.shape[-2] (HC) must be 4")
    _need(hc_fn, torch.float32, (4 * H, 24), "hc_fn")
    _need(hc_scale, torch.float32, (3,), "hc_scale")
    _need(hc_base, torch.float32, (24,), "hc_base")
    dev = R.device
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if y is None else y
    pre = torch.empty((T, 4), dtype=torch.float32, device=dev) if pre is None else pre
    post = torch.empty((T, 4), dtype=torch.float32, device=dev) if post is None else post
    comb = torch.empty((T, 4, 4), dtype=torch.float32, device=dev) if comb is None else comb
    _need(y, torch.bfloat16, (T, H), "y")
    _need(pre, torch.float32, (T, 4), "pre")
    _need(post, torch.float32, None, "post")
    _need(comb, torch.float32, (T, 4, 4), "comb")
    nws = workspace_bytes(T, H)
    if workspace is None and nws > 0:
        workspace = torch.empty(nws, dtype=torch.uint8, device=dev)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    p = params if params is not None else default_params()
    st = lib().mhc_pre_with_path(_ptr(R), _ptr(hc_fn), _ptr(hc_scale), _ptr(hc_base), _ptr(y),
                                 _ptr(pre), _ptr(post), _ptr(comb), _ptr(workspace), wsb, T, H,
                                 ctypes.byref(p), int(path), _stream(stream))
    _check(st, "mhc_pre")
    return y, pre, post, comb


def _pre_outputs(R, y, pre, post, comb):
    import torch
    T, _, H = R.shape
    dev = R.device
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if y is None else y
    pre = torch.empty((T, 4), dtype=torch.float32, device=dev) if pre is None else pre
    post = torch.empty((T, 4), dtype=torch.float32, device=dev) if post is None else post
    comb = torch.empty((T, 4, 4), dtype=torch.float32, device=dev) if comb is None else comb
    _need(y, torch.bfloat16, (T, H), "y")
    _need(pre, torch.float32, (T, 4), "pre")
    _need(post, torch.float32, None, "post")
    if post.numel() != T * 4:
        raise ValueError("post must hold T*4 values ([T,4] or [T,4,1])")
    _need(comb, torch.float32, (T, 4, 4), "comb")
    return y, pre, post, comb


def pre_big_fuse(dot_mix, sqrsum, R, hc_scale, hc_base, k: int, *, num_splits: int = 1, y=None,
                 pre=None, post=None, comb=None, params: Params | None = None, stream=None):
    """Pre-map from an external projection: dot_mix [num_splits,T,24] (or [T,24] for one split)
    and sqrsum [num_splits,T] (or [T]) fp32 partials, R [T,4,H] bf16, RMS denominator k.
    Returns (y, pre, post, comb)."""
    import torch
    _need(R, torch.bfloat16, None, "R")
    T, hc, H = R.shape
    if hc != 4:
        raise ValueError("R.shape[-2] (HC) must be 4")
    _need(dot_mix, torch.float32, None, "dot_mix")
    _need(sqrsum, torch.float32, None, "sqrsum")
    if dot_mix.numel() != num_splits * T * 24 or sqrsum.numel() != num_splits * T:
        raise ValueError("dot_mix must hold num_splits*T*24 values and sqrsum num_splits*T")
    _need(hc_scale, torch.float32, (3,), "hc_scale")
    _need(hc_base, torch.float32, (24,), "hc_base")
    y, pre, post, comb = _pre_outputs(R, y, pre, post, comb)
    p = params if params is not None else default_params()
    st = lib().mhc_pre_big_fuse(_ptr(dot_mix), _ptr(sqrsum), int(num_splits), int(k), _ptr(R),
                                _ptr(hc_scale), _ptr(hc_base), _ptr(y), _ptr(pre), _ptr(post),
                                _ptr(comb), T, H, ctypes.byref(p), _stream(stream))
    _check(st, "mhc_pre_big_fuse")
    return y, pre, post, comb


def pre_big_fuse_with_prenorm(dot_mix, R, hc_scale, hc_base, *, y=None, pre=None, post=None,
                              comb=None, params: Params | None = None, stream=None):
    """Pre-map from an external projection dot_mix [T,24] (or [1,T,24]); the sum of squares is
    formed from R and the RMS denominator is 4H. Returns (y, pre, post, comb)."""
    import torch
    _need(R, torch.bfloat16, None, "R")
    T, hc, H = R.shape
    if hc != 4:
        raise ValueError("R.shape[-2] (HC) must be 4")
    _need(dot_mix, torch.float32, None, "dot_mix")
    if dot_mix.numel() != T * 24:
        raise ValueError("dot_mix must hold T*24 values")
    _need(hc_scale, torch.float32, (3,), "hc_scale")
    _need(hc_base, torch.float32, (24,), "hc_base")
    y, pre, post, comb = _pre_outputs(R, y, pre, post, comb)
    p = params if params is not None else default_params()
    st = lib().mhc_pre_big_fuse_with_prenorm(_ptr(dot_mix), _ptr(R), _ptr(hc_scale),
                                             _ptr(hc_base), _ptr(y), _ptr(pre), _ptr(post),
                                             _ptr(comb), T, H, ctypes.byref(p), _stream(stream))
    _check(st, "mhc_pre_big_fuse_with_prenorm")
    return y, pre, post, comb


def post_project_splits(T: int, H: int) -> int:
    """Splits S of the partials mhc_post_project writes for (T, H); 0 when unsupported."""
    return int(lib().mhc_post_project_splits(int(T), int(H)))


def post_project(x, R, post, comb, hc_fn_next, *, out=None, dot_mix=None, sqrsum=None,
                 workspace=None, stream=None):
    """Post-map fused with the next site's projection partials. Returns (out [T,4,H] bf16,
    dot_mix [S,T,24], sqrsum [S,T]); finish the next pre-map with
    pre_big_fuse(dot_mix, sqrsum, out, ..., k=4H, num_splits=S)."""
    import torch
    _need(R, torch.bfloat16, None, "R")
    T, hc, H = R.shape
    if hc != 4:
        raise ValueError("R.shape[-2] (HC) must be 4")
    _need(x, torch.bfloat16, (T, H), "x")
    _need(post, torch.float32, None, "post")
    if post.numel() != T * 4:
        raise ValueError("post must hold T*4 values ([T,4] or [T,4,1])")
    _need(comb, torch.float32, (T, 4, 4), "comb")
    _need(hc_fn_next, torch.float32, (4 * H, 24), "hc_fn_next")
    S = post_project_splits(T, H) if T > 0 else 1
    if T > 0 and S == 0:
        raise MhcError(MHC_ERR_UNSUPPORTED, "mhc_post_project")
    dev = R.device
    out = torch.empty_like(R) if out is None else out
    dot_mix = torch.empty((S, T, 24), dtype=torch.float32, device=dev) if dot_mix is None else dot_mix
    sqrsum = torch.empty((S, T), dtype=torch.float32, device=dev) if sqrsum is None else sqrsum
    _need(out, torch.bfloat16, (T, 4, H), "out")
    _need(dot_mix, torch.float32, (S, T, 24), "dot_mix")
    _need(sqrsum, torch.float32, (S, T), "sqrsum")
    nws = int(lib().mhc_post_project_workspace_bytes(T, H))
    if workspace is None and nws > 0:
        workspace = torch.empty(nws, dtype=torch.uint8, device=dev)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().mhc_post_project(_ptr(x), _ptr(R), _ptr(post), _ptr(comb), _ptr(out),
                                _ptr(hc_fn_next), _ptr(dot_mix), _ptr(sqrsum), _ptr(workspace),
                                wsb, T, H, _stream(stream))
    _check(st, "mhc_post_project")
    return out, dot_mix, sqrsum


def post_backward(d_out, x, R, post, comb, *, stream=None):
    """Backward of the post-map. Returns (d_x [T,H] bf16, d_R [T,4,H] bf16, d_post [T,4],
    d_comb [T,4,4] fp32)."""
    import torch
    _need(R, torch.bfloat16, None, "R")
    T, hc, H = R.shape
    _need(d_out, torch.bfloat16, (T, 4, H), "d_out")
    _need(x, torch.bfloat16, (T, H), "x")
    _need(post, torch.float32, None, "post")
    _need(comb, torch.float32, (T, 4, 4), "comb")
    dev = R.device
    d_x = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    d_R = torch.empty_like(R)
    d_post = torch.empty((T, 4), dtype=torch.float32, device=dev)
    d_comb = torch.empty((T, 4, 4), dtype=torch.float32, device=dev)
    st = lib().mhc_post_backward(_ptr(d_out), _ptr(x), _ptr(R), _ptr(post), _ptr(comb),
                                 _ptr(d_x), _ptr(d_R), _ptr(d_post), _ptr(d_comb), T, H,
                                 _stream(stream))
    _check(st, "mhc_post_backward")
    return d_x, d_R, d_post, d_comb


def pre_backward(R, hc_fn, hc_scale, hc_base, *, d_y=None, d_pre=None, d_post=None, d_comb=None,
                 params: Params | None = None, workspace=None, stream=None):
    """Backward of the pre-map from the upstream gradients (any may be None). Returns
    (d_R [T,4,H] bf16, d_hc_fn [4H,24], d_scale [3], d_base [24] fp32)."""
    import torch
    _need(R, torch.bfloat16, None, "R")
    T, hc, H = R.shape
    _need(hc_fn, torch.float32, (4 * H, 24), "hc_fn")
    _need(hc_scale, torch.float32, (3,), "hc_scale")
    _need(hc_base, torch.float32, (24,), "hc_base")
    if d_y is not None:
        _need(d_y, torch.bfloat16, (T, H), "d_y")
    for name, tsr, n in (("d_pre", d_pre, 4), ("d_post", d_post, 4), ("d_comb", d_comb, 16)):
        if tsr is not None:
            _need(tsr, torch.float32, None, name)
            if tsr.numel() != T * n:
                raise ValueError(f"{name} must hold T*{n} values")
    dev = R.device
    d_R = torch.empty_like(R)
    d_W = torch.empty((4 * H, 24), dtype=torch.float32, device=dev)
    d_s = torch.empty(3, dtype=torch.float32, device=dev)
    d_b = torch.empty(24, dtype=torch.float32, device=dev)
    nws = int(lib().mhc_pre_backward_workspace_bytes(T, H))
    if workspace is None and nws > 0:
        workspace = torch.empty(nws, dtype=torch.uint8, device=dev)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    p = params if params is not None else default_params()
    st = lib().mhc_pre_backward(_ptr(d_y), _ptr(d_pre), _ptr(d_post), _ptr(d_comb), _ptr(R),
                                _ptr(hc_fn), _ptr(hc_scale), _ptr(hc_base), _ptr(d_R), _ptr(d_W),
                                _ptr(d_s), _ptr(d_b), _ptr(workspace), wsb, T, H, ctypes.byref(p),
                                _stream(stream))
    _check(st, "mhc_pre_backward")
    return d_R, d_W, d_s, d_b


def expand(hidden, *, streams=None, stream=None):
    """First-layer expand: hidden [T,H] bf16 -> streams [T,4,H] bf16 (each stream a copy)."""
    import torch
    _need(hidden, torch.bfloat16, None, "hidden")
    T, H = hidden.shape
    streams = torch.empty((T, 4, H), dtype=torch.bfloat16, device=hidden.device) \
        if streams is None else streams
    _need(streams, torch.bfloat16, (T, 4, H), "streams")
    _check(lib().mhc_expand(_ptr(hidden), _ptr(streams), T, H, _stream(stream)), "mhc_expand")
    return streams


def head_mean(R, *, y=None, stream=None):
    """Last-layer unweighted head: y [T,H] = bf16(mean of the 4 streams of R [T,4,H])."""
    import torch
    _need(R, torch.bfloat16, None, "R")
    T, hc, H = R.shape
    if hc != 4:
        raise ValueError("R.shape[-2] (HC) must be 4")
    y = torch.empty((T, H), dtype=torch.bfloat16, device=R.device) if y is None else y
    _need(y, torch.bfloat16, (T, H), "y")
    _check(lib().mhc_head_mean(_ptr(R), _ptr(y), T, H, _stream(stream)), "mhc_head_mean")
    return y


def head_workspace_bytes(T: int, H: int) -> int:
    return int(lib().mhc_head_workspace_bytes(int(T), int(H)))


def head(R, hc_fn, hc_scale, hc_base, *, norm_eps: float = 1e-6, hc_eps: float = 1e-6, y=None,
         weights=None, workspace=None, stream=None):
    """Last-layer weighted head: R [T,4,H] bf16, hc_fn [4H,4], hc_scale [1], hc_base [4] fp32.
    Returns (y [T,H] bf16, weights [T,4] fp32)."""
    import torch
    _need(R, torch.bfloat16, None, "R")
    T, hc, H = R.shape
    if hc != 4:
        raise ValueError("R.shape[-2] (HC) must be 4")
    _need(hc_fn, torch.float32, (4 * H, 4), "hc_fn")
    _need(hc_scale, torch.float32, (1,), "hc_scale")
    _need(hc_base, torch.float32, (4,), "hc_base")
    dev = R.device
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if y is None else y
    weights = torch.empty((T, 4), dtype=torch.float32, device=dev) if weights is None else weights
    _need(y, torch.bfloat16, (T, H), "y")
    _need(weights, torch.float32, (T, 4), "weights")
    nws = head_workspace_bytes(T, H)
    if workspace is None and nws > 0:
        workspace = torch.empty(nws, dtype=torch.uint8, device=dev)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().mhc_head(_ptr(R), _ptr(hc_fn), _ptr(hc_scale), _ptr(hc_base), _ptr(y),
                        _ptr(weights), _ptr(workspace), wsb, T, H, float(norm_eps), float(hc_eps),
                        _stream(stream))
    _check(st, "mhc_head")
    return y, weights


def post(x, R, post, comb, *, out=None, path: int = PATH_AUTO, stream=None):
    """Post-map. x [T,H], R [T,4,H] bf16; post [T,4] (or [T,4,1]), comb [T,4,4] fp32.
    Returns out [T,4,H] bf16 (pass out=R to update the residual in place)."""
    import torch
    _need(R, torch.bfloat16, None, "R")
    T, hc, H = R.shape
    if hc != 4:
        raise ValueError("R.shape[-2] (HC) must be 4")
    _need(x, torch.bfloat16, (T, H), "x")
    _need(post, torch.float32, None, "post")
    if post.numel() != T * 4:
        raise ValueError("post must hold T*4 values ([T,4] or [T,4,1])")
    _need(comb, torch.float32, (T, 4, 4), "comb")
    out = torch.empty_like(R) if out is None else out
    _need(out, torch.bfloat16, (T, 4, H), "out")
    st = lib().mhc_post_with_path(_ptr(x), _ptr(R), _ptr(post), _ptr(comb), _ptr(out), T, H,
                                  int(path), _stream(stream))
    _check(st, "mhc_post")
    return out


def sinkhorn(logits, *, comb=None, iters: int = 20, eps: float = 1e-6, stream=None):
    """Standalone Sinkhorn on logits [T,4,4] fp32. Returns comb [T,4,4]."""
    import torch
    _need(logits, torch.float32, None, "logits")
    if logits.shape[-2:] != (4, 4):
        raise ValueError("logits must be [..., 4, 4]")
    T = logits.numel() // 16
    comb = torch.empty_like(logits) if comb is None else comb
    _need(comb, torch.float32, tuple(logits.shape), "comb")
    st = lib().mhc_sinkhorn(_ptr(logits), _ptr(comb), T, 0, int(iters), float(eps),
                            _stream(stream))
    _check(st, "mhc_sinkhorn")
    return comb


def device_status(stream=None) -> int:
    """Reads and clears the library's device-side status word (0, or MHC_ERR_TIMEOUT)."""
    return int(lib().mhc_device_status(_stream(stream)))


def selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Enqueues the bounded-wait health check: a kernel whose wait nothing ends gives up after
    limit_ns and records MHC_ERR_TIMEOUT in the device status word (read it with device_status)."""
    st = lib().mhc_selftest_wait_timeout(int(limit_ns), _stream(stream))
    if st != MHC_OK:
        raise MhcError(st, "mhc_selftest_wait_timeout")


def launch_count() -> int:
    """Kernel launches this process has enqueued through the library."""
    return int(lib().mhc_launch_count())


def build_library(force: bool = False) -> str:
    """Compile libmhc.so in-tree (nvcc, sm_100a)."""
    import importlib
    return importlib.import_module(__name__ + ".build").build(force=force)
