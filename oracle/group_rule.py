"""Second, independent oracle: brute force over all token pairs (NumPy float64).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

It never rolls or partitions anything. Working on the zero-padded grid of
extents Lp = ceil(L / w) * w, it lets token i attend to token j exactly when,
on every axis, ``floor((o_i - s) / w) == floor((o_j - s) / w)`` (floor
division, so coordinates below the shift get group -1). That one rule is the
shifted window plus the region mask of the "Video Swin Transformer" summary
page (Method step 5: shifted windows and the mask that blocks pairs that were
not neighbours before the roll):

* for o >= s the rolled coordinate is r = o - s and the group is the window
  index r // w; the last group (nw - 1) is the region [Lp - w, Lp - s) of the
  last window;
* for o < s the rolled coordinate wraps to r = o - s + Lp in [Lp - s, Lp), the
  region of the last window that came from the start of the grid; its group
  is -1.

So the groups are in one-to-one correspondence with (window, region) pairs,
and inside a group the relative offset used by the bias is the original one,
o_i - o_j. With zero shift the groups are the plain windows. Padded tokens
are keys with zero input, never masked. Cost grows with (Tp*Hp*Wp)^2, so use
small grids only.
"""

from __future__ import annotations

import numpy as np


def _padded_coords(Lp):
    t, h, w = np.meshgrid(np.arange(Lp[0]), np.arange(Lp[1]), np.arange(Lp[2]), indexing="ij")
    return np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1)  # (Np, 3)


def forward(x, window, shift, Wqkv, bqkv, Wproj, bproj, table, heads):
    x = np.asarray(x, dtype=np.float64)
    B, T, H, W, C = x.shape
    L = np.array([T, H, W])
    w = np.array(window)
    s = np.array(shift)
    Lp = -(-L // w) * w
    d = C // heads
    coords = _padded_coords(Lp)  # (Np, 3)
    Np = coords.shape[0]
    group = np.floor_divide(coords - s, w)  # (Np, 3)
    allowed = np.all(group[:, None, :] == group[None, :, :], axis=2)  # (Np, Np)
    delta = coords[:, None, :] - coords[None, :, :]  # query - key
    nh, nwd = 2 * w[1] - 1, 2 * w[2] - 1
    idx = (delta[..., 0] + w[0] - 1) * nh * nwd + (delta[..., 1] + w[1] - 1) * nwd + (delta[..., 2] + w[2] - 1)
    idx = np.where(allowed, idx, 0)  # offsets outside a group are never used
    real = np.all(coords < L, axis=1)
    table = np.asarray(table, dtype=np.float64)

    out = np.zeros_like(x)
    for b in range(B):
        xp = np.zeros((Np, C))
        xp[real] = x[b].reshape(-1, C)  # coords enumerate (t, h, w) row-major
        qkv = xp @ np.asarray(Wqkv, dtype=np.float64) + np.asarray(bqkv, dtype=np.float64)
        o = np.zeros((Np, C))
        for hd in range(heads):
            q = qkv[:, hd * d:(hd + 1) * d]
            k = qkv[:, C + hd * d:C + (hd + 1) * d]
            v = qkv[:, 2 * C + hd * d:2 * C + (hd + 1) * d]
            scores = q @ k.T / np.sqrt(d) + table[idx, hd]
            scores = np.where(allowed, scores, -np.inf)
            scores -= scores.max(axis=1, keepdims=True)
            p = np.exp(scores)
            p /= p.sum(axis=1, keepdims=True)
            o[:, hd * d:(hd + 1) * d] = p @ v
        y = o @ np.asarray(Wproj, dtype=np.float64) + np.asarray(bproj, dtype=np.float64)
        out[b] = y[real].reshape(T, H, W, C)
    return out
