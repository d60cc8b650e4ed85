"""Seeded synthetic inputs shared by the CUDA path, the oracle and the benchmark.

This module holds random-number generation and dtype rounding only -- none of
the layer's arithmetic. Both sides receive the very same rounded values: the
CUDA library as torch tensors of the run dtype, the oracle as float64 copies.

Recipe (stands in for Kinetics clips; no dataset is used):
  * CPU ``torch.Generator`` seeded with ``1000 * workload_index + k + seed_offset``,
    k = 0: x, 1: Wqkv, 2: Wproj, 3: table, 4: bqkv, 5: bproj;
  * "baseline" scale: x ~ N(0, 1); Wqkv, Wproj, table ~ N(0, 0.02); biases 0;
  * "sensitivity" scale (correctness only): x ~ N(0, 1); Wqkv, Wproj ~ N(0, 1/C);
    table ~ N(0, 1); biases ~ N(0, 0.1), so that dropping the mask, the bias or
    a bias vector moves the output far outside the tolerances;
  * values drawn in float32, then rounded once to the run dtype.

Block inputs (layer norm + layer + residual) add, from seeds k = 6, 7, 8: a
per-token offset ~ N(0, 0.5) added to x (so that the norm's centring matters),
gamma ~ 1 + N(0, 0.1) and beta ~ N(0, 0.1).

MLP-half inputs (layer norm + two linear layers with GELU + residual), seeds
k = 10..16: x ~ N(0, 1) plus a per-token offset ~ N(0, 0.5); gamma ~ 1 + N(0, 0.1),
beta ~ N(0, 0.1); "baseline" W1, W2 ~ N(0, 0.02) and biases 0; "sensitivity"
W1 ~ N(0, 1/C), W2 ~ N(0, 1/hidden), biases ~ N(0, 0.1).

Patch-merging inputs, seeds k = 20..24: x as for the MLP half; gamma ~ 1 + N(0, 0.1),
beta ~ N(0, 0.1) over 4C; "baseline" Wr ~ N(0, 0.02), no bias; "sensitivity"
Wr ~ N(0, 1/(4C)), br ~ N(0, 0.1).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass
class LayerInputs:
    x: torch.Tensor
    Wqkv: torch.Tensor
    bqkv: torch.Tensor
    Wproj: torch.Tensor
    bproj: torch.Tensor
    table: torch.Tensor

    def as_f64(self):
        """float64 NumPy copies of the exact (rounded) values, for the oracle."""
        return {k: getattr(self, k).to(torch.float64).numpy() for k in
                ("x", "Wqkv", "bqkv", "Wproj", "bproj", "table")}

    def to(self, device):
        return LayerInputs(*(getattr(self, k).to(device) for k in
                             ("x", "Wqkv", "bqkv", "Wproj", "bproj", "table")))


def table_rows(window) -> int:
    return (2 * window[0] - 1) * (2 * window[1] - 1) * (2 * window[2] - 1)


def _randn(shape, seed, std):
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32) * std


def make_layer_inputs(shape, heads, window, dtype="bf16", scale="baseline", seed=1000,
                      x_seed=None) -> LayerInputs:
    """Inputs for one layer call. ``shape`` = (B, T, H, W, C)."""
    B, T, H, W, C = shape
    dt = _DT[dtype]
    nt = table_rows(window)
    xs = seed if x_seed is None else x_seed
    if scale == "baseline":
        w_std, t_std, b_std = 0.02, 0.02, 0.0
    elif scale == "sensitivity":
        w_std, t_std, b_std = 1.0 / np.sqrt(C), 1.0, 0.1
    else:
        raise ValueError(scale)
    x = _randn((B, T, H, W, C), xs + 0, 1.0)
    Wqkv = _randn((C, 3 * C), seed + 1, w_std)
    Wproj = _randn((C, C), seed + 2, w_std)
    table = _randn((nt, heads), seed + 3, t_std)
    bqkv = _randn((3 * C,), seed + 4, b_std) if b_std else torch.zeros(3 * C)
    bproj = _randn((C,), seed + 5, b_std) if b_std else torch.zeros(C)
    return LayerInputs(*(t.to(dt).contiguous() for t in (x, Wqkv, bqkv, Wproj, bproj, table)))


def workload_layer_inputs(workload, layer, scale="baseline") -> LayerInputs:
    """Inputs of one layer of a named workload (see ``workloads.py``).

    The two layers of the W-MSA + SW-MSA pair get their own weights but the
    same N(0,1) input (x is seeded without the layer's offset)."""
    base = 1000 * workload.index
    return make_layer_inputs(layer.shape, layer.heads, layer.window, workload.dtype, scale,
                             seed=base + layer.seed_offset, x_seed=base)


@dataclass
class BlockInputs:
    layer: LayerInputs
    gamma: torch.Tensor
    beta: torch.Tensor

    def as_f64(self):
        d = self.layer.as_f64()
        d["gamma"] = self.gamma.to(torch.float64).numpy()
        d["beta"] = self.beta.to(torch.float64).numpy()
        return d

    def to(self, device):
        return BlockInputs(self.layer.to(device), self.gamma.to(device), self.beta.to(device))


def make_block_inputs(shape, heads, window, dtype="bf16", scale="baseline", seed=1000,
                      x_seed=None) -> BlockInputs:
    """Inputs for one call of the block's attention half (layer norm, layer, residual)."""
    B, T, H, W, C = shape
    dt = _DT[dtype]
    xs = seed if x_seed is None else x_seed
    li = make_layer_inputs(shape, heads, window, dtype, scale, seed=seed, x_seed=xs)
    offset = _randn((B, T, H, W, 1), xs + 6, 0.5)
    x = (li.x.float() + offset).to(dt).contiguous()
    gamma = (1.0 + _randn((C,), seed + 7, 0.1)).to(dt).contiguous()
    beta = _randn((C,), seed + 8, 0.1).to(dt).contiguous()
    li = LayerInputs(x, li.Wqkv, li.bqkv, li.Wproj, li.bproj, li.table)
    return BlockInputs(li, gamma, beta)


@dataclass
class MlpInputs:
    x: torch.Tensor
    gamma: torch.Tensor
    beta: torch.Tensor
    W1: torch.Tensor
    b1: torch.Tensor
    W2: torch.Tensor
    b2: torch.Tensor

    _KEYS = ("x", "gamma", "beta", "W1", "b1", "W2", "b2")

    def as_f64(self):
        return {k: getattr(self, k).to(torch.float64).numpy() for k in self._KEYS}

    def to(self, device):
        return MlpInputs(*(getattr(self, k).to(device) for k in self._KEYS))


def make_mlp_inputs(shape, hidden, dtype="bf16", scale="baseline", seed=1000) -> MlpInputs:
    """Inputs for one call of a block's MLP half. ``shape`` = (B, T, H, W, C)."""
    B, T, H, W, C = shape
    dt = _DT[dtype]
    if scale == "baseline":
        w1_std, w2_std, b_std = 0.02, 0.02, 0.0
    elif scale == "sensitivity":
        w1_std, w2_std, b_std = 1.0 / np.sqrt(C), 1.0 / np.sqrt(hidden), 0.1
    else:
        raise ValueError(scale)
    x = _randn((B, T, H, W, C), seed + 10, 1.0) + _randn((B, T, H, W, 1), seed + 11, 0.5)
    gamma = 1.0 + _randn((C,), seed + 12, 0.1)
    beta = _randn((C,), seed + 13, 0.1)
    W1 = _randn((C, hidden), seed + 14, w1_std)
    W2 = _randn((hidden, C), seed + 15, w2_std)
    b1 = _randn((hidden,), seed + 16, b_std) if b_std else torch.zeros(hidden)
    b2 = _randn((C,), seed + 17, b_std) if b_std else torch.zeros(C)
    return MlpInputs(*(t.to(dt).contiguous() for t in (x, gamma, beta, W1, b1, W2, b2)))


@dataclass
class MergeInputs:
    x: torch.Tensor
    gamma: torch.Tensor
    beta: torch.Tensor
    Wr: torch.Tensor
    br: object  # torch.Tensor or None

    def as_f64(self):
        d = {k: getattr(self, k).to(torch.float64).numpy() for k in ("x", "gamma", "beta", "Wr")}
        d["br"] = None if self.br is None else self.br.to(torch.float64).numpy()
        return d

    def to(self, device):
        return MergeInputs(self.x.to(device), self.gamma.to(device), self.beta.to(device), self.Wr.to(device),
                           None if self.br is None else self.br.to(device))


def make_merge_inputs(shape, dtype="bf16", scale="baseline", seed=1000) -> MergeInputs:
    """Inputs for one patch-merging call. ``shape`` = (B, T, H, W, C)."""
    B, T, H, W, C = shape
    dt = _DT[dtype]
    if scale == "baseline":
        w_std, b_std = 0.02, 0.0
    elif scale == "sensitivity":
        w_std, b_std = 1.0 / np.sqrt(4 * C), 0.1
    else:
        raise ValueError(scale)
    x = _randn((B, T, H, W, C), seed + 20, 1.0) + _randn((B, T, H, W, 1), seed + 21, 0.5)
    gamma = 1.0 + _randn((4 * C,), seed + 22, 0.1)
    beta = _randn((4 * C,), seed + 23, 0.1)
    Wr = _randn((4 * C, 2 * C), seed + 24, w_std)
    br = _randn((2 * C,), seed + 25, b_std).to(dt).contiguous() if b_std else None
    return MergeInputs(*(t.to(dt).contiguous() for t in (x, gamma, beta, Wr)), br)
