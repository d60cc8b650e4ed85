"""GPU parity of the fused MLP half of a block (vswin_mlp_forward: layer norm, two
linear layers with GELU, residual) against the float64 oracle's mlp_half on the same
seeded inputs. Needs a B200."""

import numpy as np
import pytest
import torch

import oracle
from shifted_window_attention_sw_b200 import vswin
from shifted_window_attention_sw_b200.inputs import make_mlp_inputs

pytestmark = pytest.mark.gpu

EPS = 1e-5
# Like the block entry: the branch (out - x) takes the layer's relative gates; out is
# x + branch rounded once to bf16, so each element may also carry half a bf16 step of
# |out| (2^-9 relative), hence 2^-8 in the elementwise gate. The branch rounds LN(x) and
# GELU(.) to bf16 as MMA operands and evaluates GELU through a tanh form within
# 1e-3 |x| of the erf form, an order below those roundings.
BRANCH_REL_L2, BRANCH_REL_MAX = 1e-2, 3e-2
ABS_MAX, ABS_MEAN = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shifted_window_attention_sw_b200 import build

    build.build()
    vswin.lib()


def _ref(a):
    return oracle.mlp_half(a["x"], a["gamma"], a["beta"], EPS, a["W1"], a["b1"], a["W2"], a["b2"])


def _gpu(inp, in_place=False):
    d = inp.to("cuda")
    out = d.x if in_place else None
    out = vswin.mlp_forward(d.x, d.gamma, d.beta, EPS, d.W1, d.b1, d.W2, d.b2, out=out)
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


MLP_CASES = [
    # (shape (B, T, H, W, C), hidden)
    ((1, 8, 14, 14, 96), 384),     # Swin-T width, hidden 4C: weights resident, 13 tiles
    ((2, 5, 9, 10, 64), 256),      # 900 tokens: a ragged last tile of 4 rows
    ((1, 8, 14, 14, 128), 512),    # Swin-B width: 64-column hidden chunks streamed through 2 stages
    ((1, 3, 5, 7, 32), 128),       # one chunk, fewer tokens than one tile
    ((1, 4, 7, 7, 96), 768),       # hidden 8C: 128-column chunks streamed
]


@pytest.mark.parametrize("shape,hidden", MLP_CASES)
@pytest.mark.parametrize("scale", ["baseline", "sensitivity"])
def test_mlp(shape, hidden, scale):
    inp = make_mlp_inputs(shape, hidden, "bf16", scale, seed=8000 + sum(shape))
    a = inp.as_f64()
    _check(_gpu(inp), _ref(a), a["x"], scale == "sensitivity")


def test_mlp_in_place():
    inp = make_mlp_inputs((2, 8, 14, 14, 96), 384, "bf16", "sensitivity", seed=8100)
    a = inp.as_f64()
    _check(_gpu(inp, in_place=True), _ref(a), a["x"], True)


@pytest.mark.parametrize("scale", ["baseline", "sensitivity"])
def test_mlp_headline_whole_tensor(scale):
    # the headline token tensor (8, 16, 56, 56, 96), hidden 4C: 3136 tiles, about 21
    # per persistent CTA, every output element against the oracle
    inp = make_mlp_inputs((8, 16, 56, 56, 96), 384, "bf16", scale, seed=8200)
    a = inp.as_f64()
    _check(_gpu(inp), _ref(a), a["x"], scale == "sensitivity")


def test_mlp_deterministic():
    d = make_mlp_inputs((2, 16, 28, 28, 96), 384, "bf16", "sensitivity", seed=8300).to("cuda")
    o1 = vswin.mlp_forward(d.x, d.gamma, d.beta, EPS, d.W1, d.b1, d.W2, d.b2)
    o2 = vswin.mlp_forward(d.x, d.gamma, d.beta, EPS, d.W1, d.b1, d.W2, d.b2)
    assert vswin.poll_error() == vswin.OK
    assert torch.equal(o1, o2)


# ------------------------------------------------------------------ whole block (eq. 1)
def _block_inputs(shape, heads, window, scale, seed):
    from shifted_window_attention_sw_b200.inputs import make_block_inputs

    b = make_block_inputs(shape, heads, window, "bf16", scale, seed=seed)
    m = make_mlp_inputs(shape, 4 * shape[-1], "bf16", scale, seed=seed + 50)
    return b, m


def _block_ref(b, m, window, shift, heads):
    a = b.as_f64()
    mm = m.as_f64()
    attn = dict(gamma=a["gamma"], beta=a["beta"], Wqkv=a["Wqkv"], bqkv=a["bqkv"], Wproj=a["Wproj"],
                bproj=a["bproj"], table=a["table"])
    mlp = dict(gamma=mm["gamma"], beta=mm["beta"], W1=mm["W1"], b1=mm["b1"], W2=mm["W2"], b2=mm["b2"])
    return a["x"], oracle.block_full_forward(a["x"], attn, mlp, window, shift, heads, eps=EPS)


def _block_gpu(b, m, window, shift, heads):
    d, md = b.to("cuda"), m.to("cuda")
    li = d.layer
    attn = dict(gamma=d.gamma, beta=d.beta, Wqkv=li.Wqkv, bqkv=li.bqkv, Wproj=li.Wproj, bproj=li.bproj,
                table=li.table)
    mlp = dict(gamma=md.gamma, beta=md.beta, W1=md.W1, b1=md.b1, W2=md.W2, b2=md.b2)
    out = vswin.block_forward(li.x, window, shift, attn, mlp, heads, eps=EPS)
    assert vswin.poll_error() == vswin.OK, vswin.last_error()
    return out.double().cpu().numpy()


@pytest.mark.parametrize("shape,heads,window,shift", [
    ((1, 8, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)),
    ((1, 12, 12, 12, 128), 4, (8, 7, 7), (4, 3, 3)),   # padding on every axis, Swin-B width
    ((2, 1, 14, 21, 64), 2, (1, 7, 7), (0, 3, 3)),     # 2D Swin special case
])
@pytest.mark.parametrize("scale", ["baseline", "sensitivity"])
def test_whole_block(shape, heads, window, shift, scale):
    b, m = _block_inputs(shape, heads, window, scale, seed=9000 + sum(shape))
    x, ref = _block_ref(b, m, window, shift, heads)
    out = _block_gpu(b, m, window, shift, heads)
    _check(out, ref, x, scale == "sensitivity")


def test_whole_block_headline_whole_tensor():
    # the headline SW-MSA layer shape as a whole block, every element against the oracle
    b, m = _block_inputs((8, 16, 56, 56, 96), 3, (8, 7, 7), "sensitivity", seed=9100)
    x, ref = _block_ref(b, m, (8, 7, 7), (4, 3, 3), 3)
    out = _block_gpu(b, m, (8, 7, 7), (4, 3, 3), 3)
    _check(out, ref, x, True)
