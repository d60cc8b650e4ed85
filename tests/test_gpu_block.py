"""GPU parity of the fused block entry (layer norm, layer, residual) against the
CPU oracle's block_forward on the same seeded inputs. Needs a B200."""

import numpy as np
import pytest
import torch

import oracle
from shifted_window_attention_sw_b200 import vswin
from shifted_window_attention_sw_b200.inputs import make_block_inputs
from shifted_window_attention_sw_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu

EPS = 1e-5
# The branch (out - x) takes the layer's gates (relative L2 <= 1e-2, max error <= 3e-2 of
# the branch's max); out itself is x + branch rounded once to bf16, so each element may
# also carry half a bf16 step of |out| (2^-9 relative): the elementwise gate allows 2^-8.
BRANCH_REL_L2, BRANCH_REL_MAX = 1e-2, 3e-2
ABS_MAX, ABS_MEAN = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shifted_window_attention_sw_b200 import build

    build.build()
    oracle.build()
    vswin.lib()


def _ref(a, window, shift, heads):
    return oracle.block_forward(a["x"], a["gamma"], a["beta"], EPS, window, shift, a["Wqkv"], a["bqkv"],
                                a["Wproj"], a["bproj"], a["table"], heads)


def _gpu(inp, window, shift, heads, in_place=False):
    d = inp.to("cuda")
    li = d.layer
    out = li.x if in_place else None
    out = vswin.block_msa_forward(li.x, window, shift, d.gamma, d.beta, EPS, li.Wqkv, li.bqkv, li.Wproj, li.bproj,
                                  li.table, heads, out=out)
    assert vswin.poll_error() == vswin.OK, vswin.last_error()
    return out.double().cpu().numpy()


def _check(out, ref, x, sensitivity):
    assert np.isfinite(out).all()
    err = np.abs(out - ref)
    assert (err <= 2.0 ** -8 * np.abs(ref) + ABS_MAX).all(), float(err.max())
    if not sensitivity:
        assert err.mean() <= ABS_MEAN, float(err.mean())
        return
    br, br_ref = out - x, ref - x
    rel_l2 = np.linalg.norm(br - br_ref) / np.linalg.norm(br_ref)
    rel_max = np.abs(br - br_ref).max() / np.abs(br_ref).max()
    assert rel_l2 <= BRANCH_REL_L2, rel_l2
    assert rel_max <= BRANCH_REL_MAX, rel_max


BLOCK_CASES = [
    # (shape, heads, window, shift)
    ((1, 8, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)),      # Swin-T width: persistent GEMMs
    ((1, 8, 14, 14, 96), 3, (8, 7, 7), (0, 0, 0)),
    ((1, 12, 12, 12, 128), 4, (8, 7, 7), (4, 3, 3)),    # pads T, H, W
    ((1, 8, 14, 14, 384), 12, (8, 7, 7), (4, 3, 3)),    # Swin-T stage-3 width: tiled GEMMs
    ((1, 8, 7, 14, 544), 17, (8, 7, 7), (4, 0, 3)),     # 17 heads: statistics for any C/32
    ((2, 1, 14, 21, 64), 2, (1, 7, 7), (0, 3, 3)),      # 2D Swin special case
    ((1, 5, 9, 10, 64), 2, (4, 4, 4), (2, 1, 3)),       # padding on every axis, generic attention kernel
]


@pytest.mark.parametrize("shape,heads,window,shift", BLOCK_CASES)
@pytest.mark.parametrize("scale", ["baseline", "sensitivity"])
def test_block(shape, heads, window, shift, scale):
    inp = make_block_inputs(shape, heads, window, "bf16", scale, seed=5000 + sum(shape))
    a = inp.as_f64()
    ref = _ref(a, window, shift, heads)
    out = _gpu(inp, window, shift, heads)
    _check(out, ref, a["x"], scale == "sensitivity")


def test_block_in_place():
    shape, heads, window, shift = (2, 16, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)
    inp = make_block_inputs(shape, heads, window, "bf16", "sensitivity", seed=5100)
    a = inp.as_f64()
    ref = _ref(a, window, shift, heads)
    out = _gpu(inp, window, shift, heads, in_place=True)
    _check(out, ref, a["x"], True)


def test_block_matches_layer_on_normalised_input():
    # With gamma = 1 and beta = 0 and x already normalised (in bf16), the branch is the
    # plain layer on that input; the two entries may differ only by their roundings.
    shape, heads, window, shift = (1, 8, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)
    inp = make_block_inputs(shape, heads, window, "bf16", "sensitivity", seed=5200)
    d = inp.to("cuda")
    li = d.layer
    ones = torch.ones_like(d.gamma)
    zeros = torch.zeros_like(d.beta)
    blk = vswin.block_msa_forward(li.x, window, shift, ones, zeros, EPS, li.Wqkv, li.bqkv, li.Wproj, li.bproj,
                                  li.table, heads)
    xn = torch.nn.functional.layer_norm(li.x.float(), (shape[-1],), eps=EPS).to(torch.bfloat16)
    lay = vswin.wmsa_forward(xn, window, shift, li.Wqkv, li.bqkv, li.Wproj, li.bproj, li.table, heads)
    assert vswin.poll_error() == vswin.OK, vswin.last_error()
    br = (blk.float() - li.x.float()).double()
    rel = (br - lay.double()).norm() / lay.double().norm()
    assert rel <= 2e-2, float(rel)


def test_block_full_size_sampled():
    # the headline workload's first layer shape as a block, sampled windows against the oracle
    wl = WORKLOADS["swin_t_s1_b8"]
    layer = wl.layers[1]
    inp = make_block_inputs(layer.shape, layer.heads, layer.window, "bf16", "sensitivity", seed=5300)
    out = _gpu(inp, layer.window, layer.shift, layer.heads)
    a = inp.as_f64()
    g = oracle.geometry(layer.T, layer.H, layer.W, layer.window, layer.shift)
    nW, nw = g["nW"], g["nw"]
    wins = sorted({0, layer.B * nW - 1, (layer.B // 2) * nW + nW // 2, nw[1] * nw[2] - 1, nW - 1})
    y = oracle.block_forward_windows(a["x"], a["gamma"], a["beta"], EPS, layer.window, layer.shift, a["Wqkv"],
                                     a["bqkv"], a["Wproj"], a["bproj"], a["table"], layer.heads, wins)
    src, _, _ = oracle.index_maps(layer.B, layer.T, layer.H, layer.W, layer.window, layer.shift)
    N = g["N"]
    flat = out.reshape(-1, layer.C)
    xf = a["x"].reshape(-1, layer.C)
    got, exp, xs = [], [], []
    for k, w in enumerate(wins):
        s = src[w * N:(w + 1) * N]
        m = s >= 0
        got.append(flat[s[m]])
        exp.append(y[k][m])
        xs.append(xf[s[m]])
    _check(np.concatenate(got), np.concatenate(exp), np.concatenate(xs), True)
    assert np.isfinite(out).all()


@pytest.mark.parametrize("scale", ["baseline", "sensitivity"])
def test_block_headline_whole_tensor(scale):
    # the headline SW-MSA layer shape as a block, every output element against the oracle
    wl = WORKLOADS["swin_t_s1_b8"]
    layer = wl.layers[1]
    inp = make_block_inputs(layer.shape, layer.heads, layer.window, "bf16", scale, seed=5400)
    a = inp.as_f64()
    out = _gpu(inp, layer.window, layer.shift, layer.heads)
    ref = _ref(a, layer.window, layer.shift, layer.heads)
    _check(out, ref, a["x"], scale == "sensitivity")
