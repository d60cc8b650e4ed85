"""Algorithmic work of one layer call: FLOPs, compulsory bytes, exponentials.

Per window of K tokens and width D the layer costs 4*K*D^2 + 2*K^2*D
multiply-adds: the q, k, v and output projections (4*K*D^2) plus QK^T and PV
(2*K^2*D) ("Swin Transformer" tutorial page, section 3.1, complexity table).
Here that is counted per layer, batched over all windows:

    FLOPs = 2*tok*C*3C + 2*tok*C*C + 4*windows*N^2*C

with tok = real tokens (a padded slot needs no projection GEMM: its
projection is the bias) and N = P*Mh*Mw tokens per window. Masked pairs are
counted, because the method computes them; the unmasked count is reported
beside it. Compulsory bytes = read x + write out + weights + biases + table.
"""

from __future__ import annotations


def window_multiply_adds(K: int, D: int) -> int:
    return 4 * K * D * D + 2 * K * K * D


def _ceil_to(v, m):
    return -(-v // m) * m


def unmasked_pairs(T, H, W, window, shift) -> int:
    """Query/key pairs inside windows that share a region (per clip)."""
    total = 1
    for L, w, s in zip((T, H, W), window, shift):
        Lp = _ceil_to(L, w)
        nw = Lp // w
        # Pairs on this axis summed over its windows: every window but the last
        # contributes w^2; the last one, when shifted, splits into (w - s) and s.
        last = w * w if s == 0 else (w - s) ** 2 + s * s
        total *= (nw - 1) * w * w + last
    return total


def layer_work(B, T, H, W, C, heads, window, shift, elem_bytes=2):
    Lp = [_ceil_to(L, w) for L, w in zip((T, H, W), window)]
    nW = (Lp[0] // window[0]) * (Lp[1] // window[1]) * (Lp[2] // window[2])
    N = window[0] * window[1] * window[2]
    tok = B * T * H * W
    windows = B * nW
    gemm_flops = 2 * tok * C * 3 * C + 2 * tok * C * C
    attn_flops = 4 * windows * N * N * C
    nt = (2 * window[0] - 1) * (2 * window[1] - 1) * (2 * window[2] - 1)
    bytes_ = elem_bytes * (2 * tok * C + 3 * C * C + 3 * C + C * C + C + nt * heads)
    pairs = windows * N * N
    return {
        "tokens": tok,
        "windows": windows,
        "N": N,
        "gemm_flops": gemm_flops,
        "attn_flops": attn_flops,
        "flops": gemm_flops + attn_flops,
        "bytes": bytes_,
        "exps": pairs * heads,
        "pairs": pairs,
        "unmasked_pairs": B * unmasked_pairs(T, H, W, window, shift),
    }
