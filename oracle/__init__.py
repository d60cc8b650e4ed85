"""CPU oracle for the 3D (shifted-)window attention layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``; never
by the product package. It shares no code with the CUDA library.

Two independent formulations live here:

* ``forward`` -- ``vswin_oracle.cpp``, double precision, the pages' steps in
  order (pad, roll by -shift, window partition, QKV, masked
  softmax(QK^T/sqrt(d) + B)V, projection, reverse partition, roll by +shift,
  un-pad). "Video Swin Transformer" summary page, Method steps 3-6 and the
  window_msa pseudocode; eq. 2.
* ``group_rule.forward`` -- a NumPy float64 brute force over all token pairs of
  the padded grid with no roll and no partition (see that module).

Gradients of the layer (``oracle.backward``, NumPy float64) follow the same
steps per window and the chain rule back through them; they are pinned by
central finite differences of ``forward``.

The attention half of a block (``block_forward``) is written on top of
``forward`` in NumPy float64: layer norm of each token over its C channels,
the layer, and the residual add ("Video Swin Transformer" summary page, Method
step 3 and eq. 1; Video Swin code walk-through page, section 1.2: LayerNorm
comes before F.pad, so padded tokens are zeros after the norm).
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vswin_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

NO_MASK = 1
POS_ROLL = 2
NO_BIAS = 4
ROLL_THEN_PAD = 8
MASK_ADD100 = 16

_lib = None


def build(force: bool = False) -> str:
    """Compile ``vswin_oracle.cpp`` into ``liboracle.so`` (g++, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["g++", "-O2", "-std=c++17", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        lib.vswin_oracle_forward_ex.argtypes = [
            dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ip, ip, dp, dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_long, ctypes.c_int, dp,
        ]
        lib.vswin_oracle_forward_ex.restype = ctypes.c_int
        lib.vswin_oracle_forward_windows.argtypes = [
            dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ip, ip, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_long), ctypes.c_int, dp, ctypes.c_int,
        ]
        lib.vswin_oracle_forward_windows.restype = ctypes.c_int
        lib.vswin_oracle_index_maps.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ip, ip, ip, ip, ip,
        ]
        lib.vswin_oracle_index_maps.restype = ctypes.c_int
        lib.vswin_oracle_max_threads.argtypes = [ctypes.c_int]
        lib.vswin_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _iarr(v) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(v, dtype=np.int32).reshape(3))


def _iptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def max_threads(nthreads: int = 0) -> int:
    """OpenMP threads the oracle uses with ``nthreads`` (0 = library default)."""
    return int(_load().vswin_oracle_max_threads(int(nthreads)))


def geometry(T, H, W, window, shift=(0, 0, 0)):
    """Padded extents, windows per axis, windows per clip and tokens per window."""
    L = (T, H, W)
    Lp = tuple(-(-L[a] // window[a]) * window[a] for a in range(3))
    nw = tuple(Lp[a] // window[a] for a in range(3))
    return {
        "Lp": Lp,
        "nw": nw,
        "nW": nw[0] * nw[1] * nw[2],
        "N": window[0] * window[1] * window[2],
    }


def forward(x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, flags=0, nthreads=0,
            probe=None):
    """Layer forward in double precision.

    x: (B,T,H,W,C); Wqkv [C][3C]; bqkv [3C]; Wproj [C][C]; bproj [C];
    table [(2P-1)(2Mh-1)(2Mw-1)][heads]. window/shift are taken literally.
    probe=(b, window_index, head) additionally returns that head's N x N
    attention probabilities.
    """
    lib = _load()
    x = _f64(x)
    B, T, H, W, C = x.shape
    g = geometry(T, H, W, window, shift)
    N = g["N"]
    out = np.empty_like(x)
    w_arr, s_arr = _iarr(window), _iarr(shift)
    Wqkv, bqkv, Wproj, bproj, table = map(_f64, (Wqkv, bqkv, Wproj, bproj, table))
    assert Wqkv.shape == (C, 3 * C) and bqkv.shape == (3 * C,)
    assert Wproj.shape == (C, C) and bproj.shape == (C,)
    nt = (2 * window[0] - 1) * (2 * window[1] - 1) * (2 * window[2] - 1)
    assert table.shape == (nt, heads)
    probs = None
    pb, pw, ph = -1, -1, -1
    if probe is not None:
        pb, pw, ph = probe
        probs = np.zeros((N, N), dtype=np.float64)
    rc = lib.vswin_oracle_forward_ex(
        _dptr(x), B, T, H, W, C, heads, _iptr(w_arr), _iptr(s_arr),
        _dptr(Wqkv), _dptr(bqkv), _dptr(Wproj), _dptr(bproj), _dptr(table), _dptr(out),
        int(flags), int(nthreads), pb, pw, ph, _dptr(probs) if probs is not None else None,
    )
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (status {rc})")
    if probe is not None:
        return out, probs
    return out


def forward_windows(x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, windows, nthreads=0):
    """Per-window outputs (len(windows), N, C) in slot order for the listed global
    windows b * nW + w (no reverse partition): the same arithmetic as ``forward``."""
    lib = _load()
    x = _f64(x)
    B, T, H, W, C = x.shape
    N = geometry(T, H, W, window, shift)["N"]
    wl = np.ascontiguousarray(np.asarray(windows, dtype=np.int64))
    y = np.empty((wl.size, N, C), dtype=np.float64)
    w_arr, s_arr = _iarr(window), _iarr(shift)
    Wqkv, bqkv, Wproj, bproj, table = map(_f64, (Wqkv, bqkv, Wproj, bproj, table))
    rc = lib.vswin_oracle_forward_windows(
        _dptr(x), B, T, H, W, C, heads, _iptr(w_arr), _iptr(s_arr), _dptr(Wqkv), _dptr(bqkv),
        _dptr(Wproj), _dptr(bproj), _dptr(table), wl.ctypes.data_as(ctypes.POINTER(ctypes.c_long)),
        int(wl.size), _dptr(y), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (status {rc})")
    return y


def index_maps(B, T, H, W, window, shift):
    """(win_src[B*nW*N], region[nW*N], bias_idx[N*N]) as int32 arrays."""
    lib = _load()
    g = geometry(T, H, W, window, shift)
    N, nW = g["N"], g["nW"]
    win_src = np.empty(B * nW * N, dtype=np.int32)
    region = np.empty(nW * N, dtype=np.int32)
    bias_idx = np.empty(N * N, dtype=np.int32)
    w_arr, s_arr = _iarr(window), _iarr(shift)
    rc = lib.vswin_oracle_index_maps(B, T, H, W, _iptr(w_arr), _iptr(s_arr),
                                     _iptr(win_src), _iptr(region), _iptr(bias_idx))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (status {rc})")
    return win_src, region, bias_idx


LN_EPS = 1e-5  # torch.nn.LayerNorm's default; the code walk-through page names nn.LayerNorm


def layer_norm(x, gamma, beta, eps=LN_EPS):
    """Layer norm of each token over its last axis, in float64.

    (x - mean) / sqrt(var + eps) * gamma + beta with the biased variance
    (mean of squared deviations), as torch.nn.LayerNorm computes it. "Video
    Swin Transformer" summary page, Method step 3 and eq. 1 (LN).
    """
    x = _f64(x)
    gamma, beta = _f64(gamma), _f64(beta)
    mean = x.mean(axis=-1, keepdims=True)
    dev = x - mean
    var = (dev * dev).mean(axis=-1, keepdims=True)
    return dev / np.sqrt(var + float(eps)) * gamma + beta


def block_forward(x, gamma, beta, eps, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, flags=0,
                  nthreads=0):
    """Attention half of a Video Swin block in float64: x + layer(LN(x)).

    "Video Swin Transformer" summary page, eq. 1 (z_hat = 3D(S)W-MSA(LN(z)) + z)
    and the block pseudocode; the layer is ``forward`` with the same arguments.
    """
    x = _f64(x)
    y = layer_norm(x, gamma, beta, eps)
    return x + forward(y, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, flags=flags,
                       nthreads=nthreads)


def block_forward_windows(x, gamma, beta, eps, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads,
                          windows, nthreads=0):
    """``block_forward`` restricted to the listed windows (flat b * nW + w).

    Returns (len(windows), N, C): for each window slot that holds a real
    token, that token's block output; padding slots hold the layer's value
    there without a residual (they are not outputs of the block). The norm
    is per token, so normalising the whole tensor first is exact.
    """
    x = _f64(x)
    y = layer_norm(x, gamma, beta, eps)
    o = forward_windows(y, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, windows, nthreads=nthreads)
    B, T, H, W, C = x.shape
    src, _, _ = index_maps(B, T, H, W, window, shift)
    N = o.shape[1]
    flat = x.reshape(-1, C)
    for k, w in enumerate(windows):
        s = src[int(w) * N:(int(w) + 1) * N]
        m = s >= 0
        o[k][m] += flat[s[m]]
    return o


def gelu(x):
    """x * Phi(x), Phi the standard normal CDF (the erf form of torch.nn.GELU)."""
    from scipy.special import erf

    x = _f64(x)
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def mlp_half(z, gamma, beta, eps, W1, b1, W2, b2):
    """Second half of a block in float64: z + GELU(LN(z) W1 + b1) W2 + b2.

    "Video Swin Transformer" summary page, Method step 3 and eq. 1 (layer norm,
    a two-layer MLP with GELU, residual add). W1 [C][hidden], W2 [hidden][C];
    the pages do not give the hidden width (Swin's models use 4C).
    """
    z = _f64(z)
    W1, b1, W2, b2 = map(_f64, (W1, b1, W2, b2))
    y = layer_norm(z, gamma, beta, eps)
    return z + gelu(y @ W1 + b1) @ W2 + b2


def block_full_forward(x, attn, mlp, window, shift, heads, eps=LN_EPS):
    """One whole Video Swin block in float64 (eq. 1): the attention half
    (``block_forward``) then ``mlp_half``. ``attn`` = dict(gamma, beta, Wqkv, bqkv,
    Wproj, bproj, table); ``mlp`` = dict(gamma, beta, W1, b1, W2, b2)."""
    z = block_forward(x, attn["gamma"], attn["beta"], eps, window, shift, attn["Wqkv"], attn["bqkv"],
                      attn["Wproj"], attn["bproj"], attn["table"], heads)
    return mlp_half(z, mlp["gamma"], mlp["beta"], eps, mlp["W1"], mlp["b1"], mlp["W2"], mlp["b2"])


def patch_merge_gather(x):
    """The 2x2 spatial neighbour concatenation of patch merging, in float64.

    "Video Swin Transformer" summary page, Method step 2 (each 2x2 group of
    spatial neighbours, 4C values; no temporal merging) and the code walk-through
    page, section 1.2 (PatchMerging: interval sampling of H and W, channels x4).
    The pages do not fix the order of the four neighbours inside the 4C vector
    nor what happens at an odd H or W. Readings taken: neighbour (dh, dw) of
    merged token (i, j) is x[2i + dh, 2j + dw] and sits at channels
    [(2 dw + dh) C, (2 dw + dh + 1) C) -- the order (0,0), (1,0), (0,1), (1,1) --
    and an odd H or W is zero-padded by one row or column at the high end (the
    padding convention of the window partition). Returns (B, T, ceil(H/2),
    ceil(W/2), 4C).
    """
    x = _f64(x)
    B, T, H, W, C = x.shape
    Hp, Wp = H + H % 2, W + W % 2
    xp = np.zeros((B, T, Hp, Wp, C))
    xp[:, :, :H, :W] = x
    parts = []
    for dw in (0, 1):
        for dh in (0, 1):
            parts.append(xp[:, :, dh::2, dw::2, :])
    return np.concatenate(parts, axis=-1)


def patch_merge(x, gamma, beta, eps, Wr, br=None):
    """Patch merging between stages in float64: LN over the 4C concatenation of each
    2x2 spatial neighbourhood, then one linear layer 4C -> 2C.

    "Video Swin Transformer" summary page, Method step 2 (concatenate each 2x2
    group of spatial neighbours and project 4C to 2C with a linear layer); the
    code walk-through page, section 1.2 (PatchMerging: nn.LayerNorm then
    nn.Linear(4 * dim, 2 * dim)). Wr is [4C][2C]; ``br`` is an optional bias
    (the pages do not say whether the projection has one; None = none).
    """
    z = layer_norm(patch_merge_gather(x), gamma, beta, eps)
    y = z @ _f64(Wr)
    if br is not None:
        y = y + _f64(br)
    return y
