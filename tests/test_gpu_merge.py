"""GPU parity of patch merging (vswin_patch_merge_forward: 2x2 spatial neighbour
concatenation, layer norm over 4C, linear 4C -> 2C) against the float64 oracle's
patch_merge on the same seeded inputs. Needs a B200."""

import numpy as np
import pytest
import torch

import oracle
from shifted_window_attention_sw_b200 import vswin
from shifted_window_attention_sw_b200.inputs import make_merge_inputs

pytestmark = pytest.mark.gpu

EPS = 1e-5
# One GEMM with the norm folded into bf16 weights and the output rounded once to bf16:
# the layer's relative gates apply (relative L2 error 1e-2, max error 3e-2 of the max).
REL_L2, REL_MAX = 1e-2, 3e-2
ABS_MAX, ABS_MEAN = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shifted_window_attention_sw_b200 import build

    build.build()
    vswin.lib()


def _run(shape, scale, seed):
    inp = make_merge_inputs(shape, "bf16", scale, seed=seed)
    a = inp.as_f64()
    ref = oracle.patch_merge(a["x"], a["gamma"], a["beta"], EPS, a["Wr"], a["br"])
    d = inp.to("cuda")
    out = vswin.patch_merge_forward(d.x, d.gamma, d.beta, EPS, d.Wr, d.br)
    assert vswin.poll_error() == vswin.OK, vswin.last_error()
    return out.double().cpu().numpy(), ref


MERGE_CASES = [
    (1, 8, 14, 14, 96),     # Swin-T stage 1 -> 2 width
    (2, 3, 9, 11, 64),      # odd H and W: zero-padded neighbours
    (1, 4, 8, 8, 384),      # Swin-T stage 3 -> 4: 2C = 768, three N tiles of 256
    (1, 2, 5, 6, 32),       # fewer merged tokens than one tile
    (1, 2, 6, 6, 160),      # 2C = 320: N tiles of 160
]


@pytest.mark.parametrize("shape", MERGE_CASES)
@pytest.mark.parametrize("scale", ["baseline", "sensitivity"])
def test_patch_merge(shape, scale):
    out, ref = _run(shape, scale, 11000 + sum(shape))
    assert out.shape == ref.shape
    assert np.isfinite(out).all()
    err = out - ref
    rel_l2 = np.linalg.norm(err) / np.linalg.norm(ref)
    rel_max = np.abs(err).max() / np.abs(ref).max()
    assert rel_l2 <= REL_L2, rel_l2
    assert rel_max <= REL_MAX, rel_max
    if scale == "baseline":
        assert np.abs(err).max() <= ABS_MAX and np.abs(err).mean() <= ABS_MEAN


def test_patch_merge_column_slices_several_tiles_per_cta():
    # Swin-T stage 2 -> 3 at batch 8: 2C = 384 in four resident 96-column weight
    # slices, 200 row tiles of 9 lines x 14 merged tokens (TMA gather) over 37 CTAs
    # per slice (five or six tiles each, both accumulators and the statistics ring
    # reused), every element against the oracle
    out, ref = _run((8, 16, 28, 28, 192), "sensitivity", 11600)
    err = out - ref
    assert np.linalg.norm(err) / np.linalg.norm(ref) <= REL_L2
    assert np.abs(err).max() / np.abs(ref).max() <= REL_MAX


def test_patch_merge_odd_sizes_several_tiles_per_cta():
    # odd H and W (the cp.async gather, zero-filled neighbours on the last row and
    # column): 784 row tiles on 148 CTAs, every element against the oracle
    out, ref = _run((8, 16, 55, 55, 96), "sensitivity", 11650)
    err = out - ref
    assert np.linalg.norm(err) / np.linalg.norm(ref) <= REL_L2
    assert np.abs(err).max() / np.abs(ref).max() <= REL_MAX


def test_patch_merge_widest_channels_tiled_kernel():
    # C = 1536: even 16-column slices would be 192 of them, more than the SMs (and one
    # of 6144 rows would not leave room for four A stages), so the tiled kernel runs
    out, ref = _run((1, 2, 3, 4, 1536), "baseline", 11700)
    err = out - ref
    assert np.linalg.norm(err) / np.linalg.norm(ref) <= REL_L2
    assert np.abs(err).max() / np.abs(ref).max() <= REL_MAX


def test_patch_merge_headline_whole_tensor():
    # the headline stage-1 token tensor (8, 16, 56, 56, 96) -> (8, 16, 28, 28, 192): 896
    # tiles of 4 lines x 28 merged tokens (TMA gather), every element against the oracle
    out, ref = _run((8, 16, 56, 56, 96), "sensitivity", 11500)
    err = out - ref
    assert np.linalg.norm(err) / np.linalg.norm(ref) <= REL_L2
    assert np.abs(err).max() / np.abs(ref).max() <= REL_MAX
