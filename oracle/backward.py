"""Gradients of the (shifted-)window attention layer, NumPy float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): imported by ``tests/``
alone. It shares no code with the CUDA library.

For a loss L whose gradient with respect to the layer output is ``dy``,
``backward`` returns dL/dx, dL/dWqkv, dL/dbqkv, dL/dWproj, dL/dbproj and
dL/dtable of the layer ``oracle.forward`` computes. It runs the forward's
steps per window in the pages' order ("Video Swin Transformer" summary page,
Method steps 4-6, the window_msa pseudocode and eq. 2: gather the window from
the rolled, padded grid, qkv = X Wqkv + bqkv, per head
P = softmax(q k^T / sqrt(d) + B) over the keys of the query's region,
O = P v, y = O Wproj + bproj, scatter back), then the chain rule through them
in reverse. The one step that is not a product rule is the softmax:
dS = P * (dP - rowsum(dP * P)), which is zero wherever P is (masked pairs).
Window maps (source token of every slot, region id, bias-table row of every
pair) come from ``oracle.index_maps``, so the roll / pad / partition is the
one the forward oracle uses.

Readings: padded slots are keys with zero input (their q / k / v are the
biases), so they receive gradient through bqkv but none reaches x; the table
gradient of a head is the sum of dS over every (window, query, key) pair
that reads that table row.
"""

from __future__ import annotations

import numpy as np

from . import geometry, index_maps


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _window_maps(B, T, H, W, window, shift):
    g = geometry(T, H, W, window, shift)
    src, region, bias_idx = index_maps(B, T, H, W, window, shift)
    return g, src, region, bias_idx.reshape(g["N"], g["N"])


def _window_forward(X, allowed, bidx, Wqkv, bqkv, table, heads):
    """qkv and the per-head probabilities and outputs of one window."""
    N, C = X.shape
    d = C // heads
    qkv = X @ Wqkv + bqkv
    O = np.zeros((N, C))
    probs = []
    for h in range(heads):
        q = qkv[:, h * d:(h + 1) * d]
        k = qkv[:, C + h * d:C + (h + 1) * d]
        v = qkv[:, 2 * C + h * d:2 * C + (h + 1) * d]
        S = q @ k.T / np.sqrt(d) + table[bidx, h]
        S = np.where(allowed, S, -np.inf)
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P /= P.sum(axis=1, keepdims=True)
        O[:, h * d:(h + 1) * d] = P @ v
        probs.append(P)
    return qkv, O, probs


def forward(x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads):
    """The layer, recomputed the way ``backward`` does (for checking that the
    gradient is taken of the same function as ``oracle.forward``)."""
    x = _f64(x)
    Wqkv, bqkv, Wproj, bproj, table = map(_f64, (Wqkv, bqkv, Wproj, bproj, table))
    B, T, H, W, C = x.shape
    g, src, region, bidx = _window_maps(B, T, H, W, window, shift)
    N, nW = g["N"], g["nW"]
    xf = x.reshape(-1, C)
    out = np.zeros_like(xf)
    for wi in range(B * nW):
        s = src[wi * N:(wi + 1) * N]
        real = s >= 0
        X = np.zeros((N, C))
        X[real] = xf[s[real]]
        reg = region[(wi % nW) * N:(wi % nW + 1) * N]
        allowed = reg[:, None] == reg[None, :]
        _, O, _ = _window_forward(X, allowed, bidx, Wqkv, bqkv, table, heads)
        y = O @ Wproj + bproj
        out[s[real]] = y[real]
    return out.reshape(x.shape)


def backward(x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads, dy):
    """(dx, dWqkv, dbqkv, dWproj, dbproj, dtable) for output gradient ``dy``."""
    x, dy = _f64(x), _f64(dy)
    Wqkv, bqkv, Wproj, bproj, table = map(_f64, (Wqkv, bqkv, Wproj, bproj, table))
    B, T, H, W, C = x.shape
    assert dy.shape == x.shape
    d = C // heads
    g, src, region, bidx = _window_maps(B, T, H, W, window, shift)
    N, nW = g["N"], g["nW"]
    xf, dyf = x.reshape(-1, C), dy.reshape(-1, C)
    dx = np.zeros_like(xf)
    dWqkv, dbqkv = np.zeros_like(Wqkv), np.zeros_like(bqkv)
    dWproj, dbproj = np.zeros_like(Wproj), np.zeros_like(bproj)
    dtable = np.zeros_like(table)
    flat_idx = bidx.ravel()
    for wi in range(B * nW):
        s = src[wi * N:(wi + 1) * N]
        real = s >= 0
        X = np.zeros((N, C))
        X[real] = xf[s[real]]
        reg = region[(wi % nW) * N:(wi % nW + 1) * N]
        allowed = reg[:, None] == reg[None, :]
        qkv, O, probs = _window_forward(X, allowed, bidx, Wqkv, bqkv, table, heads)
        # output projection and scatter: padding slots are not outputs (zero gradient)
        dY = np.zeros((N, C))
        dY[real] = dyf[s[real]]
        dWproj += O.T @ dY
        dbproj += dY.sum(axis=0)
        dO = dY @ Wproj.T
        dqkv = np.zeros((N, 3 * C))
        for h in range(heads):
            q = qkv[:, h * d:(h + 1) * d]
            k = qkv[:, C + h * d:C + (h + 1) * d]
            v = qkv[:, 2 * C + h * d:2 * C + (h + 1) * d]
            P = probs[h]
            dOh = dO[:, h * d:(h + 1) * d]
            dP = dOh @ v.T
            dS = P * (dP - (dP * P).sum(axis=1, keepdims=True))
            dqkv[:, h * d:(h + 1) * d] = dS @ k / np.sqrt(d)
            dqkv[:, C + h * d:C + (h + 1) * d] = dS.T @ q / np.sqrt(d)
            dqkv[:, 2 * C + h * d:2 * C + (h + 1) * d] = P.T @ dOh
            np.add.at(dtable[:, h], flat_idx, dS.ravel())
        dWqkv += X.T @ dqkv
        dbqkv += dqkv.sum(axis=0)
        dX = dqkv @ Wqkv.T
        dx[s[real]] += dX[real]  # every token sits in exactly one window slot
    return dx.reshape(x.shape), dWqkv, dbqkv, dWproj, dbproj, dtable
