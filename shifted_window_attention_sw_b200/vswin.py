"""ctypes binding of ``libvswin.so`` (``include/vswin.h``): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; PyTorch only owns
device memory and streams. There is no fallback: if the library is missing
or a call fails, a ``VswinError`` is raised.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# VSWIN_LIBRARY may name another build of the same library (the in-tree
# libvswin_debug.so, built with VSWIN_DEBUG_BOUNDS) to load instead.
LIB_PATH = os.environ.get("VSWIN_LIBRARY") or os.path.join(_PKG, "libvswin.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_NO_MEMORY, ERR_BOUNDS = range(7)
INJECT_CUDA, INJECT_ALLOC = 1, 2

# Every symbol include/vswin.h declares.
EXPORTS = (
    "vswin_wmsa_forward",
    "vswin_wmsa_forward_f32",
    "vswin_wmsa_forward_host",
    "vswin_wmsa_index_maps",
    "vswin_clamp_window",
    "vswin_last_error",
    "vswin_poll_error",
    "vswin_launch_count",
    "vswin_set_wait_limit_ns",
    "vswin_selftest_timeout",
    "vswin_version",
    "vswin_profile_enable",
    "vswin_profile_collect",
    "vswin_wmsa_forward_noalloc",
    "vswin_set_exact_softmax",
    "vswin_block_msa_forward",
    "vswin_wmsa_backward_f32",
    "vswin_wmsa_backward",
    "vswin_mlp_forward",
    "vswin_block_forward",
    "vswin_patch_merge_forward",
    "vswin_test_inject_failure",
    "vswin_debug_plant_row",
    "vswin_debug_bounds_enabled",
)

KERNEL_KINDS = ("qkv_gemm", "attention", "proj_gemm", "other", "mlp", "attention_bwd")


class VswinError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"vswin status {status}: {message}")
        self.status = status


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_IP = ctypes.POINTER(ctypes.c_int)


def lib():
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise VswinError(-1, f"{LIB_PATH} is missing: build it with "
                                 "`python -m shifted_window_attention_sw_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        layer = [_P, _I, _I, _I, _I, _I, _I, _IP, _IP, _P, _P, _P, _P, _P, _P, _P]
        for name in ("vswin_wmsa_forward", "vswin_wmsa_forward_f32", "vswin_wmsa_forward_host",
                     "vswin_wmsa_forward_noalloc"):
            fn = getattr(L, name)
            fn.argtypes = layer
            fn.restype = _I
        L.vswin_block_msa_forward.argtypes = layer[:9] + [_P, _P, ctypes.c_float] + layer[9:]
        L.vswin_block_msa_forward.restype = _I
        L.vswin_wmsa_backward_f32.argtypes = layer[:15] + [_P] * 6 + [_P]  # ..., dy, six gradients, stream
        L.vswin_wmsa_backward_f32.restype = _I
        L.vswin_wmsa_backward.argtypes = layer[:15] + [_P] * 6 + [_P]
        L.vswin_wmsa_backward.restype = _I
        L.vswin_mlp_forward.argtypes = [_P, _I, _I, _I, _I, _I, _I, _P, _P, ctypes.c_float, _P, _P, _P, _P, _P,
                                        _P]
        L.vswin_mlp_forward.restype = _I
        L.vswin_block_forward.argtypes = (layer[:9] + [_P, _P] + [_P] * 5 + [_P, _P, _I] + [_P] * 4 +
                                          [ctypes.c_float, _P, _P])
        L.vswin_block_forward.restype = _I
        L.vswin_patch_merge_forward.argtypes = [_P, _I, _I, _I, _I, _I, _P, _P, ctypes.c_float, _P, _P, _P, _P]
        L.vswin_patch_merge_forward.restype = _I
        L.vswin_wmsa_index_maps.argtypes = [_I, _I, _I, _I, _IP, _IP, _P, _P, _P, _P]
        L.vswin_wmsa_index_maps.restype = _I
        L.vswin_clamp_window.argtypes = [_I, _I, _I, _IP, _IP, _IP, _IP]
        L.vswin_clamp_window.restype = _I
        L.vswin_last_error.argtypes = []
        L.vswin_last_error.restype = ctypes.c_char_p
        L.vswin_poll_error.argtypes = [_P]
        L.vswin_poll_error.restype = _I
        L.vswin_launch_count.argtypes = []
        L.vswin_launch_count.restype = ctypes.c_ulonglong
        L.vswin_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.vswin_set_wait_limit_ns.restype = None
        L.vswin_set_exact_softmax.argtypes = [_I]
        L.vswin_set_exact_softmax.restype = None
        L.vswin_selftest_timeout.argtypes = [_P]
        L.vswin_selftest_timeout.restype = _I
        L.vswin_profile_enable.argtypes = [_I]
        L.vswin_profile_enable.restype = _I
        L.vswin_profile_collect.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_ulonglong), _I]
        L.vswin_profile_collect.restype = _I
        L.vswin_version.argtypes = []
        L.vswin_version.restype = _I
        L.vswin_test_inject_failure.argtypes = [_I, _I]
        L.vswin_test_inject_failure.restype = _I
        L.vswin_debug_plant_row.argtypes = [ctypes.c_longlong, _I]
        L.vswin_debug_plant_row.restype = _I
        L.vswin_debug_bounds_enabled.argtypes = []
        L.vswin_debug_bounds_enabled.restype = _I
        _lib = L
    return _lib


def last_error() -> str:
    return lib().vswin_last_error().decode()


def _check(status):
    if status != OK:
        raise VswinError(status, last_error())


def _i3(v):
    v = tuple(int(a) for a in v)
    if len(v) != 3:
        raise ValueError("window and shift need 3 entries")
    return (ctypes.c_int * 3)(*v)


def _stream_handle(stream, device=None):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _layer_call(fn, x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, out, stream, device=None):
    # the library launches on the current device, so make the tensors' device current
    B, T, H, W, C = x.shape
    dev = device or x.device
    with torch.cuda.device(dev):
        _check(fn(_ptr(x), B, T, H, W, C, int(heads), _i3(window), _i3(shift), _ptr(Wqkv), _ptr(bqkv),
                  _ptr(Wproj), _ptr(bproj), _ptr(table), _ptr(out), _stream_handle(stream, dev)))
    return out


def _prep(x, tensors, dtype, device=None):
    """dtype and contiguity of every tensor; with ``device``, that every tensor is a
    CUDA tensor on that device. The library reads raw pointers, so a host tensor or
    one on another GPU must be refused here."""
    for name, t in tensors.items():
        if t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if device is not None:
        for name, t in tensors.items():
            if not t.is_cuda or t.device != device:
                raise ValueError(f"{name} must be a CUDA tensor on {device}, got {t.device}")


def _table_rows(window):
    w = tuple(int(a) for a in window)
    if len(w) != 3:
        raise ValueError("window and shift need 3 entries")
    return (2 * w[0] - 1) * (2 * w[1] - 1) * (2 * w[2] - 1)


def _check_shapes(x, window, heads, Wqkv=None, bqkv=None, Wproj=None, bproj=None, table=None, **same_as_x):
    """Shapes the header fixes for a layer on x (B, T, H, W, C): Wqkv [C][3C], bqkv [3C],
    Wproj [C][C], bproj [C], bias_table [(2P-1)(2Mh-1)(2Mw-1)][heads]; every tensor in
    ``same_as_x`` has x's shape. The library trusts these sizes, so a short buffer would
    be read or written past its end."""
    if x.dim() != 5:
        raise ValueError(f"x must be (B, T, H, W, C), got shape {tuple(x.shape)}")
    C = x.shape[-1]
    want = {"Wqkv": (Wqkv, (C, 3 * C)), "bqkv": (bqkv, (3 * C,)), "Wproj": (Wproj, (C, C)),
            "bproj": (bproj, (C,)), "bias_table": (table, (_table_rows(window), int(heads)))}
    for name, (t, shape) in want.items():
        if t is not None and tuple(t.shape) != shape:
            raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
    for name, t in same_as_x.items():
        if t is not None and t.shape != x.shape:
            raise ValueError(f"{name} must have the shape of x {tuple(x.shape)}, got {tuple(t.shape)}")


def _layer_args(x, window, heads, dtype, Wqkv, bqkv, Wproj, bproj, table, out, **more):
    tensors = dict(x=x, Wqkv=Wqkv, bqkv=bqkv, Wproj=Wproj, bproj=bproj, table=table, out=out, **more)
    _prep(x, tensors, dtype, x.device)
    _check_shapes(x, window, heads, Wqkv, bqkv, Wproj, bproj, table, out=out)


def wmsa_forward(x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, out=None, stream=None):
    """bf16 layer forward on the GPU (tcgen05 path). All tensors bf16 on one CUDA device."""
    if out is None:
        out = torch.empty_like(x)
    _layer_args(x, window, heads, torch.bfloat16, Wqkv, bqkv, Wproj, bproj, table, out)
    return _layer_call(lib().vswin_wmsa_forward, x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, out,
                       stream)


def block_msa_forward(x, window, shift, gamma, beta, eps, Wqkv, bqkv, Wproj, bproj, table, heads, out=None,
                      stream=None):
    """bf16 forward of a block's attention half, out = x + layer(LN(x)), with the
    norm and the residual fused into the layer's kernels. ``out`` may be ``x``."""
    if out is None:
        out = torch.empty_like(x)
    _layer_args(x, window, heads, torch.bfloat16, Wqkv, bqkv, Wproj, bproj, table, out, gamma=gamma, beta=beta)
    B, T, H, W, C = x.shape
    for name, t in (("gamma", gamma), ("beta", beta)):
        if tuple(t.shape) != (C,):
            raise ValueError(f"{name} must have shape ({C},), got {tuple(t.shape)}")
    with torch.cuda.device(x.device):
        _check(lib().vswin_block_msa_forward(
            _ptr(x), B, T, H, W, C, int(heads), _i3(window), _i3(shift), _ptr(gamma), _ptr(beta), float(eps),
            _ptr(Wqkv), _ptr(bqkv), _ptr(Wproj), _ptr(bproj), _ptr(table), _ptr(out),
            _stream_handle(stream, x.device)))
    return out


def mlp_forward(x, gamma, beta, eps, W1, b1, W2, b2, out=None, stream=None):
    """bf16 forward of a block's MLP half, out = x + GELU(LN(x) W1 + b1) W2 + b2, as one
    fused kernel. W1 [C][hidden], W2 [hidden][C]. ``out`` may be ``x``."""
    if out is None:
        out = torch.empty_like(x)
    _prep(x, dict(x=x, gamma=gamma, beta=beta, W1=W1, b1=b1, W2=W2, b2=b2, out=out), torch.bfloat16, x.device)
    if x.dim() != 5:
        raise ValueError(f"x must be (B, T, H, W, C), got shape {tuple(x.shape)}")
    B, T, H, W, C = x.shape
    if W1.dim() != 2 or W1.shape[0] != C:
        raise ValueError(f"W1 must have shape ({C}, hidden), got {tuple(W1.shape)}")
    hidden = W1.shape[1]
    want = {"gamma": (gamma, (C,)), "beta": (beta, (C,)), "b1": (b1, (hidden,)), "W2": (W2, (hidden, C)),
            "b2": (b2, (C,)), "out": (out, tuple(x.shape))}
    for name, (t, shape) in want.items():
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
    with torch.cuda.device(x.device):
        _check(lib().vswin_mlp_forward(_ptr(x), B, T, H, W, C, int(hidden), _ptr(gamma), _ptr(beta), float(eps),
                                       _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(out),
                                       _stream_handle(stream, x.device)))
    return out


def block_forward(x, window, shift, attn, mlp, heads, eps=1e-5, out=None, stream=None):
    """bf16 forward of a whole block: z = x + layer(LN1(x)), out = z + MLP(LN2(z)).
    ``attn`` = dict(gamma, beta, Wqkv, bqkv, Wproj, bproj, table); ``mlp`` = dict(gamma, beta,
    W1, b1, W2, b2). ``out`` may be ``x``."""
    if out is None:
        out = torch.empty_like(x)
    _layer_args(x, window, heads, torch.bfloat16, attn["Wqkv"], attn["bqkv"], attn["Wproj"], attn["bproj"],
                attn["table"], out, gamma1=attn["gamma"], beta1=attn["beta"], gamma2=mlp["gamma"], beta2=mlp["beta"],
                W1=mlp["W1"], b1=mlp["b1"], W2=mlp["W2"], b2=mlp["b2"])
    B, T, H, W, C = x.shape
    hidden = mlp["W1"].shape[1] if mlp["W1"].dim() == 2 else -1
    want = {"gamma1": (attn["gamma"], (C,)), "beta1": (attn["beta"], (C,)), "gamma2": (mlp["gamma"], (C,)),
            "beta2": (mlp["beta"], (C,)), "W1": (mlp["W1"], (C, hidden)), "b1": (mlp["b1"], (hidden,)),
            "W2": (mlp["W2"], (hidden, C)), "b2": (mlp["b2"], (C,))}
    for name, (t, shape) in want.items():
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
    with torch.cuda.device(x.device):
        _check(lib().vswin_block_forward(
            _ptr(x), B, T, H, W, C, int(heads), _i3(window), _i3(shift), _ptr(attn["gamma"]), _ptr(attn["beta"]),
            _ptr(attn["Wqkv"]), _ptr(attn["bqkv"]), _ptr(attn["Wproj"]), _ptr(attn["bproj"]), _ptr(attn["table"]),
            _ptr(mlp["gamma"]), _ptr(mlp["beta"]), int(hidden), _ptr(mlp["W1"]), _ptr(mlp["b1"]), _ptr(mlp["W2"]),
            _ptr(mlp["b2"]), float(eps), _ptr(out), _stream_handle(stream, x.device)))
    return out


def patch_merge_forward(x, gamma, beta, eps, Wr, br=None, out=None, stream=None):
    """bf16 patch merging: LN over each 2x2 spatial neighbourhood's 4C values, then
    Wr [4C][2C] (+ br). x (B, T, H, W, C) -> (B, T, ceil(H/2), ceil(W/2), 2C)."""
    if x.dim() != 5:
        raise ValueError(f"x must be (B, T, H, W, C), got shape {tuple(x.shape)}")
    B, T, H, W, C = x.shape
    oshape = (B, T, (H + 1) // 2, (W + 1) // 2, 2 * C)
    if out is None:
        out = torch.empty(oshape, dtype=x.dtype, device=x.device)
    tensors = dict(x=x, gamma=gamma, beta=beta, Wr=Wr, out=out)
    if br is not None:
        tensors["br"] = br
    _prep(x, tensors, torch.bfloat16, x.device)
    want = {"gamma": (gamma, (4 * C,)), "beta": (beta, (4 * C,)), "Wr": (Wr, (4 * C, 2 * C)), "out": (out, oshape)}
    if br is not None:
        want["br"] = (br, (2 * C,))
    for name, (t, shape) in want.items():
        if tuple(t.shape) != shape:
            raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
    with torch.cuda.device(x.device):
        _check(lib().vswin_patch_merge_forward(_ptr(x), B, T, H, W, C, _ptr(gamma), _ptr(beta), float(eps),
                                               _ptr(Wr), _ptr(br), _ptr(out), _stream_handle(stream, x.device)))
    return out


def wmsa_backward_f32(x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, dy, stream=None):
    """fp32 gradients (dx, dWqkv, dbqkv, dWproj, dbproj, dtable) of the layer for output
    gradient ``dy``. All tensors float32 on one CUDA device."""
    _prep(x, dict(x=x, Wqkv=Wqkv, bqkv=bqkv, Wproj=Wproj, bproj=bproj, table=table, dy=dy), torch.float32,
          x.device)
    _check_shapes(x, window, heads, Wqkv, bqkv, Wproj, bproj, table, dy=dy)
    outs = [torch.empty_like(t) for t in (x, Wqkv, bqkv, Wproj, bproj, table)]
    B, T, H, W, C = x.shape
    with torch.cuda.device(x.device):
        _check(lib().vswin_wmsa_backward_f32(
            _ptr(x), B, T, H, W, C, int(heads), _i3(window), _i3(shift), _ptr(Wqkv), _ptr(bqkv), _ptr(Wproj),
            _ptr(bproj), _ptr(table), _ptr(dy), *[_ptr(o) for o in outs], _stream_handle(stream, x.device)))
    return tuple(outs)


def wmsa_backward(x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, dy, stream=None):
    """bf16 backward on the tensor cores: gradients (dx bf16; dWqkv, dbqkv, dWproj, dbproj,
    dtable float32) of the layer for output gradient ``dy``. Inputs bfloat16 on one CUDA
    device, as for wmsa_forward."""
    _prep(x, dict(x=x, Wqkv=Wqkv, bqkv=bqkv, Wproj=Wproj, bproj=bproj, table=table, dy=dy), torch.bfloat16,
          x.device)
    _check_shapes(x, window, heads, Wqkv, bqkv, Wproj, bproj, table, dy=dy)
    dx = torch.empty_like(x)
    grads = [torch.empty(t.shape, dtype=torch.float32, device=x.device) for t in (Wqkv, bqkv, Wproj, bproj, table)]
    B, T, H, W, C = x.shape
    with torch.cuda.device(x.device):
        _check(lib().vswin_wmsa_backward(
            _ptr(x), B, T, H, W, C, int(heads), _i3(window), _i3(shift), _ptr(Wqkv), _ptr(bqkv), _ptr(Wproj),
            _ptr(bproj), _ptr(table), _ptr(dy), _ptr(dx), *[_ptr(t) for t in grads], _stream_handle(stream, x.device)))
    return (dx, *grads)


def wmsa_forward_noalloc(x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, out=None, stream=None):
    """bf16 layer forward that allocates no device memory: the library's fixed
    32 MiB scratch array is used instead (see include/vswin.h). ``out`` should be
    passed in by callers that cannot allocate; if it is None a tensor is created."""
    if out is None:
        out = torch.empty_like(x)
    _layer_args(x, window, heads, torch.bfloat16, Wqkv, bqkv, Wproj, bproj, table, out)
    return _layer_call(lib().vswin_wmsa_forward_noalloc, x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads,
                       out, stream)


def wmsa_forward_f32(x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, out=None, stream=None):
    """fp32 layer forward on the GPU (FP32 FMA path). All tensors float32 on one CUDA device."""
    if out is None:
        out = torch.empty_like(x)
    _layer_args(x, window, heads, torch.float32, Wqkv, bqkv, Wproj, bproj, table, out)
    return _layer_call(lib().vswin_wmsa_forward_f32, x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads,
                       out, stream)


def wmsa_forward_host(x_host, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, out_host, stream=None):
    """bf16 forward with x and out in host memory (copies inside the call; synchronises)."""
    _prep(x_host, dict(x_host=x_host, out_host=out_host), torch.bfloat16)
    for name, t in (("x_host", x_host), ("out_host", out_host)):
        if t.is_cuda:
            raise ValueError(f"{name} must be a host tensor")
    dev = Wqkv.device
    _prep(x_host, dict(Wqkv=Wqkv, bqkv=bqkv, Wproj=Wproj, bproj=bproj, table=table), torch.bfloat16, dev)
    _check_shapes(x_host, window, heads, Wqkv, bqkv, Wproj, bproj, table, out_host=out_host)
    return _layer_call(lib().vswin_wmsa_forward_host, x_host, window, shift, Wqkv, bqkv, Wproj, bproj, table,
                       heads, out_host, stream, dev)


def index_maps(B, T, H, W, window, shift, device="cuda", stream=None):
    """(win_src, region, bias_idx) as int32 device tensors."""
    nW = 1
    N = 1
    for L, w in zip((T, H, W), window):
        nW *= -(-L // w)
        N *= w
    win_src = torch.empty(B * nW * N, dtype=torch.int32, device=device)
    region = torch.empty(nW * N, dtype=torch.int32, device=device)
    bias_idx = torch.empty(N * N, dtype=torch.int32, device=device)
    dev = win_src.device
    if not win_src.is_cuda:
        raise ValueError(f"index maps are written on a CUDA device, got {dev}")
    with torch.cuda.device(dev):
        _check(lib().vswin_wmsa_index_maps(B, T, H, W, _i3(window), _i3(shift), _ptr(win_src), _ptr(region),
                                           _ptr(bias_idx), _stream_handle(stream, dev)))
    return win_src, region, bias_idx


def clamp_window(T, H, W, window, shift):
    wo = (ctypes.c_int * 3)()
    so = (ctypes.c_int * 3)()
    _check(lib().vswin_clamp_window(T, H, W, _i3(window), _i3(shift), wo, so))
    return tuple(wo), tuple(so)


def poll_error(stream=None) -> int:
    """Synchronise and return the device error status (0 = OK, 4 = a kernel wait gave up,
    6 = an index check of a VSWIN_DEBUG_BOUNDS build failed)."""
    return int(lib().vswin_poll_error(_stream_handle(stream)))


def launch_count() -> int:
    return int(lib().vswin_launch_count())


def set_wait_limit_ns(ns: int) -> None:
    lib().vswin_set_wait_limit_ns(int(ns))


def set_exact_softmax(on: bool) -> None:
    """Test hook: route every query row of the bf16 (P,7,7) kernel through its exact softmax path."""
    lib().vswin_set_exact_softmax(1 if on else 0)


def selftest_timeout(stream=None) -> None:
    _check(lib().vswin_selftest_timeout(_stream_handle(stream)))


def profile_enable(on: bool) -> None:
    _check(lib().vswin_profile_enable(1 if on else 0))


def profile_collect():
    """{kind: (total ms, launches)} for the launches recorded since the last collect."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_ulonglong * n)()
    _check(lib().vswin_profile_collect(ms, cnt, n))
    return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(KERNEL_KINDS)}


def version() -> int:
    return int(lib().vswin_version())


def inject_failure(kind: int, count: int = 1) -> None:
    """Test hook: the next `count` entry calls fail as a CUDA call would (INJECT_CUDA) or
    the next `count` scratch allocations fail (INJECT_ALLOC); count 0 clears."""
    _check(lib().vswin_test_inject_failure(int(kind), int(count)))


def debug_bounds_enabled() -> bool:
    return bool(lib().vswin_debug_bounds_enabled())


def debug_plant_row(slot: int, token: int) -> None:
    """Test hook of VSWIN_DEBUG_BOUNDS builds: every following bf16 layer forward
    overwrites its row-table entry for layer slot `slot` with `token` (slot < 0: off)."""
    _check(lib().vswin_debug_plant_row(int(slot), int(token)))
