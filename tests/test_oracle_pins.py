"""Pins for the CPU oracle: what the pages and the mathematics fix, independent
of the oracle's own code. CPU only."""

import json
import os

import numpy as np
import pytest
import torch

from shifted_window_attention_sw_b200.accounting import layer_work, window_multiply_adds
from shifted_window_attention_sw_b200.inputs import make_layer_inputs, table_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_values.json")


def _inputs(shape, heads, window, scale="sensitivity", seed=77):
    return make_layer_inputs(shape, heads, window, "f32", scale, seed=seed).as_f64()


def _run(oracle_mod, a, window, shift, heads, **kw):
    return oracle_mod.forward(a["x"], window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"],
                              a["table"], heads, **kw)


# ---- P1: identity window ---------------------------------------------------------------------
def test_p1_identity_window(oracle_mod):
    # window (1,1,1): every window holds one token, its softmax is exactly 1, so the layer
    # reduces to out = (x Wv + bv) Wproj + bproj, Wv = columns [2C, 3C) of Wqkv.
    shape, heads = (2, 3, 4, 5, 16), 2
    a = _inputs(shape, heads, (1, 1, 1))
    out = _run(oracle_mod, a, (1, 1, 1), (0, 0, 0), heads)
    C = shape[-1]
    v = a["x"] @ a["Wqkv"][:, 2 * C:] + a["bqkv"][2 * C:]
    ref = v @ a["Wproj"] + a["bproj"]
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


# ---- P2: global-attention limit ----------------------------------------------------------------
def test_p2_global_limit_matches_sdpa(oracle_mod):
    # Window = whole volume, shift 0, zero table: textbook multi-head attention, checked
    # against torch's scaled_dot_product_attention in float64.
    shape, heads = (2, 2, 3, 4, 24), 3
    window = shape[1:4]
    a = _inputs(shape, heads, window)
    a["table"] = np.zeros_like(a["table"])
    out = _run(oracle_mod, a, window, (0, 0, 0), heads)
    B, C = shape[0], shape[-1]
    d = C // heads
    x = torch.from_numpy(a["x"]).reshape(B, -1, C)
    qkv = x @ torch.from_numpy(a["Wqkv"]) + torch.from_numpy(a["bqkv"])
    q, k, v = (qkv[..., i * C:(i + 1) * C].reshape(B, -1, heads, d).transpose(1, 2) for i in range(3))
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v)
    o = o.transpose(1, 2).reshape(B, -1, C)
    ref = (o @ torch.from_numpy(a["Wproj"]) + torch.from_numpy(a["bproj"])).reshape(shape).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_p2_global_limit_with_bias_matches_brute_force(oracle_mod):
    # Same limit with a nonzero table: every pair offset indexes the table directly.
    from oracle import group_rule

    shape, heads = (1, 3, 3, 4, 16), 2
    window = shape[1:4]
    a = _inputs(shape, heads, window)
    out = _run(oracle_mod, a, window, (0, 0, 0), heads)
    ref = group_rule.forward(a["x"], window, (0, 0, 0), a["Wqkv"], a["bqkv"], a["Wproj"],
                             a["bproj"], a["table"], heads)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


# ---- P3: group-rule brute force ----------------------------------------------------------------
@pytest.mark.parametrize(
    "shape,heads,window,shift",
    [
        ((1, 8, 14, 14, 32), 1, (8, 7, 7), (4, 3, 3)),   # cfg-1 geometry, shifted
        ((1, 8, 14, 14, 32), 1, (8, 7, 7), (0, 0, 0)),
        ((2, 5, 9, 10, 16), 2, (4, 4, 4), (2, 1, 3)),    # padding on every axis, partial shifts
        ((1, 6, 10, 7, 16), 2, (4, 3, 7), (0, 2, 0)),    # shift on one axis only
        ((1, 12, 8, 8, 16), 1, (8, 7, 7), (4, 3, 3)),    # T pads 12 -> 16, H/W pad 8 -> 14
        ((1, 1, 14, 14, 16), 2, (1, 7, 7), (0, 3, 3)),   # 2D Swin special case
    ],
)
def test_p3_group_rule(oracle_mod, shape, heads, window, shift):
    from oracle import group_rule

    a = _inputs(shape, heads, window)
    out = _run(oracle_mod, a, window, shift, heads)
    ref = group_rule.forward(a["x"], window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"],
                             a["table"], heads)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-11)


# ---- P4: roll/partition inverse ------------------------------------------------------------------
@pytest.mark.parametrize(
    "B,T,H,W,window,shift",
    [(2, 16, 14, 14, (8, 7, 7), (4, 3, 3)), (1, 12, 40, 40, (8, 7, 7), (4, 3, 3)),
     (1, 5, 9, 10, (4, 4, 4), (2, 1, 3)), (1, 8, 7, 7, (8, 7, 7), (4, 0, 0))],
)
def test_p4_window_source_is_a_bijection(oracle_mod, B, T, H, W, window, shift):
    win_src, region, bias_idx = oracle_mod.index_maps(B, T, H, W, window, shift)
    real = win_src[win_src >= 0]
    assert np.array_equal(np.sort(real), np.arange(B * T * H * W))
    g = oracle_mod.geometry(T, H, W, window, shift)
    assert int((win_src < 0).sum()) == B * g["nW"] * g["N"] - B * T * H * W
    # gather then scatter through the map gives x back bit for bit
    x = np.random.default_rng(0).standard_normal((B * T * H * W, 3))
    windows = np.zeros((win_src.size, 3))
    windows[win_src >= 0] = x[real]
    back = np.zeros_like(x)
    back[real] = windows[win_src >= 0]
    assert np.array_equal(back, x)


@pytest.mark.parametrize(
    "B,T,H,W,window,shift",
    [(1, 16, 14, 14, (8, 7, 7), (4, 3, 3)), (2, 5, 9, 10, (4, 4, 4), (2, 1, 3)),
     (1, 12, 40, 40, (8, 7, 7), (4, 3, 3))],
)
def test_p4_map_matches_closed_form(oracle_mod, B, T, H, W, window, shift):
    # The oracle builds the map by explicit pad + roll + partition of an index tensor. The
    # closed form: slot p of window wi sits at rolled coordinate r = wi*w + p, which holds
    # original coordinate o = (r + s) mod Lp; o >= L on any axis is padding.
    win_src, region, _ = oracle_mod.index_maps(B, T, H, W, window, shift)
    g = oracle_mod.geometry(T, H, W, window, shift)
    Lp, nw, N = g["Lp"], g["nw"], g["N"]
    L = (T, H, W)
    expect = np.empty_like(win_src)
    k = 0
    for b in range(B):
        for wt in range(nw[0]):
            for wh in range(nw[1]):
                for ww in range(nw[2]):
                    for pt in range(window[0]):
                        for ph in range(window[1]):
                            for pw in range(window[2]):
                                o = [(r + s) % lp for r, s, lp in
                                     zip((wt * window[0] + pt, wh * window[1] + ph, ww * window[2] + pw), shift, Lp)]
                                if all(o[a] < L[a] for a in range(3)):
                                    expect[k] = ((b * T + o[0]) * H + o[1]) * W + o[2]
                                else:
                                    expect[k] = -1
                                k += 1
    assert np.array_equal(win_src, expect)


# ---- P5: softmax rows --------------------------------------------------------------------------
def test_p5_softmax_rows(oracle_mod):
    shape, heads, window, shift = (1, 8, 14, 14, 32), 1, (8, 7, 7), (4, 3, 3)
    a = _inputs(shape, heads, window)
    g = oracle_mod.geometry(*shape[1:4], window, shift)
    last = g["nW"] - 1  # the last window of the clip carries all three axis splits
    _, probs = _run(oracle_mod, a, window, shift, heads, probe=(0, last, 0))
    np.testing.assert_allclose(probs.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    _, region, _ = oracle_mod.index_maps(1, *shape[1:4], window, shift)
    reg = region[last * g["N"]:(last + 1) * g["N"]]
    masked = reg[:, None] != reg[None, :]
    assert masked.any()
    assert np.all(probs[masked] == 0.0)
    assert np.all(probs[~masked] > 0.0)


# ---- P6: bias index ----------------------------------------------------------------------------
def test_p6_bias_index(oracle_mod):
    window = (8, 7, 7)
    _, _, bias_idx = oracle_mod.index_maps(1, 8, 7, 7, window, (0, 0, 0))
    N = 392
    idx = bias_idx.reshape(N, N)
    assert idx.min() >= 0 and idx.max() < 15 * 13 * 13 == table_rows(window)
    assert np.all(np.diag(idx) == 7 * 169 + 6 * 13 + 6)  # zero offset = centre row 1267
    assert np.all(idx + idx.T == 2534)                     # opposite offsets mirror around it
    # every one of the 2535 offsets occurs
    assert np.unique(idx).size == 2535


# ---- P7: shift 0 has no mask ---------------------------------------------------------------------
def test_p7_no_shift_no_mask(oracle_mod):
    shape, heads, window = (1, 8, 14, 14, 16), 2, (8, 7, 7)
    a = _inputs(shape, heads, window)
    ref = _run(oracle_mod, a, window, (0, 0, 0), heads)
    out = _run(oracle_mod, a, window, (0, 0, 0), heads, flags=oracle_mod.NO_MASK)
    assert np.array_equal(out, ref)
    _, region, _ = oracle_mod.index_maps(1, *shape[1:4], window, (0, 0, 0))
    assert np.all(region == 0)


# ---- P8: translation equivariance of W-MSA ------------------------------------------------------
def test_p8_window_translation_equivariance(oracle_mod):
    shape, heads, window = (1, 8, 14, 14, 16), 2, (4, 7, 7)
    a = _inputs(shape, heads, window)
    ref = _run(oracle_mod, a, window, (0, 0, 0), heads)
    rolled = dict(a)
    rolled["x"] = np.roll(a["x"], (4, 7, 0), axis=(1, 2, 3))
    out = _run(oracle_mod, rolled, window, (0, 0, 0), heads)
    np.testing.assert_allclose(out, np.roll(ref, (4, 7, 0), axis=(1, 2, 3)), rtol=0, atol=1e-13)


# ---- P9: batch independence ---------------------------------------------------------------------
def test_p9_batch_independence(oracle_mod):
    shape, heads, window, shift = (2, 8, 7, 14, 16), 2, (8, 7, 7), (4, 3, 3)
    a = _inputs(shape, heads, window)
    a["x"][1] = a["x"][0]
    out = _run(oracle_mod, a, window, shift, heads)
    assert np.array_equal(out[0], out[1])
    b = dict(a)
    b["x"] = a["x"].copy()
    b["x"][1] = np.random.default_rng(1).standard_normal(b["x"][1].shape)
    out2 = _run(oracle_mod, b, window, shift, heads)
    assert np.array_equal(out2[0], out[0])
    assert not np.allclose(out2[1], out[1])


# ---- P10: 2D reduction ----------------------------------------------------------------------------
def test_p10_two_d_swin(oracle_mod):
    with open(GOLDEN) as f:
        gold = json.load(f)["windows_2d"]
    H, W, M = gold["H"], gold["W"], gold["M"]
    g = oracle_mod.geometry(1, H, W, (1, M, M), (0, 3, 3))
    assert g["nW"] == gold["windows"] and g["N"] == gold["tokens_per_window"]
    from oracle import group_rule

    shape, heads = (1, 1, 14, 21, 16), 2
    a = _inputs(shape, heads, (1, 7, 7))
    out = _run(oracle_mod, a, (1, 7, 7), (0, 3, 3), heads)
    ref = group_rule.forward(a["x"], (1, 7, 7), (0, 3, 3), a["Wqkv"], a["bqkv"], a["Wproj"],
                             a["bproj"], a["table"], heads)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-11)


# ---- Mutants: each plausible slip moves the answer; -100 does not -------------------------------
def test_mutants_are_distinguishable(oracle_mod):
    # H and W pad 12 -> 14. (With only T padded 12 -> 16 and s = P/2 the two pad/roll orders
    # happen to form the same groups, so that shape cannot tell them apart.)
    shape, heads, window, shift = (1, 12, 12, 12, 32), 1, (8, 7, 7), (4, 3, 3)
    a = _inputs(shape, heads, window)
    ref = _run(oracle_mod, a, window, shift, heads)
    scale = np.abs(ref).max()
    for flag in (oracle_mod.NO_MASK, oracle_mod.POS_ROLL, oracle_mod.NO_BIAS, oracle_mod.ROLL_THEN_PAD):
        mut = _run(oracle_mod, a, window, shift, heads, flags=flag)
        assert np.abs(mut - ref).max() > 0.05 * scale, flag
    add100 = _run(oracle_mod, a, window, shift, heads, flags=oracle_mod.MASK_ADD100)
    np.testing.assert_allclose(add100, ref, rtol=0, atol=1e-14 * max(scale, 1.0))


def test_oracle_rejects_bad_arguments(oracle_mod):
    a = _inputs((1, 4, 7, 7, 16), 2, (4, 7, 7))
    with pytest.raises(ValueError):
        _run(oracle_mod, a, (4, 7, 7), (4, 0, 0), 2)  # shift must be < window


# ---- Page values (golden) ----------------------------------------------------------------------
def test_golden_flop_example():
    with open(GOLDEN) as f:
        gold = json.load(f)
    fe = gold["flop_example"]
    assert 4 * fe["K"] * fe["d"] ** 2 == fe["term_4Kd2"]
    assert 2 * fe["K"] ** 2 * fe["d"] == fe["term_2K2d"]
    assert window_multiply_adds(fe["K"], fe["d"]) == fe["per_window_multiply_adds"]
    assert round(fe["windows"] * window_multiply_adds(fe["K"], fe["d"]) / 1e6) == fe["total_approx_millions"]
    vt = gold["vit_terms"]
    assert round(2 * vt["N"] ** 2 * vt["D"] / 1e6) == vt["term_2N2D_approx_millions"]
    # layer accounting, one window of K tokens and width d: FLOPs = 2 x multiply-adds
    w = layer_work(1, 1, 7, 7, fe["d"], 1, (1, 7, 7), (0, 0, 0))
    assert w["flops"] == 2 * window_multiply_adds(49, fe["d"])


def test_golden_geometry(oracle_mod):
    with open(GOLDEN) as f:
        gold = json.load(f)
    lab = gold["windows_lab"]
    assert oracle_mod.geometry(1, lab["H"], lab["W"], (1, lab["M"], lab["M"]))["nW"] == lab["windows"]
    vt = gold["video_tokens"]
    tok = [vt["frames"] // 2, vt["height"] // 4, vt["width"] // 4]
    assert tok == vt["tokens"]
    assert oracle_mod.geometry(*tok, vt["window"])["nW"] == vt["windows_per_clip"]
    bt = gold["bias_table"]
    assert table_rows(bt["window"]) == bt["rows"]
    hs = gold["half_shift"]
    assert [w // 2 for w in hs["window"]] == hs["shift"]


def test_unmasked_fraction_matches_oracle_regions(oracle_mod):
    # accounting.unmasked_pairs (closed form) against a count over the oracle's region map
    for T, H, W, window, shift in [(16, 56, 56, (8, 7, 7), (4, 3, 3)), (12, 40, 40, (8, 7, 7), (4, 3, 3)),
                                   (16, 14, 14, (8, 7, 7), (4, 3, 3)), (5, 9, 10, (4, 4, 4), (2, 1, 3))]:
        _, region, _ = oracle_mod.index_maps(1, T, H, W, window, shift)
        g = oracle_mod.geometry(T, H, W, window, shift)
        reg = region.reshape(g["nW"], g["N"])
        count = sum(int((r[:, None] == r[None, :]).sum()) for r in reg)
        assert layer_work(1, T, H, W, 8, 1, window, shift)["unmasked_pairs"] == count


# ---- block (layer norm + layer + residual) -------------------------------------------------------
def _block_inputs(shape, heads, window, seed=88):
    from shifted_window_attention_sw_b200.inputs import make_block_inputs

    return make_block_inputs(shape, heads, window, "f32", "sensitivity", seed=seed).as_f64()


def _run_block(oracle_mod, a, window, shift, heads, eps=1e-5):
    return oracle_mod.block_forward(a["x"], a["gamma"], a["beta"], eps, window, shift, a["Wqkv"], a["bqkv"],
                                    a["Wproj"], a["bproj"], a["table"], heads)


def test_b1_layer_norm_matches_torch(oracle_mod):
    # the norm against the library routine (float64, biased variance, eps inside the root)
    a = _block_inputs((2, 3, 4, 5, 24), 2, (2, 2, 2))
    for eps in (1e-5, 1e-2):
        ref = torch.nn.functional.layer_norm(torch.from_numpy(a["x"]), (24,), torch.from_numpy(a["gamma"]),
                                             torch.from_numpy(a["beta"]), eps).numpy()
        np.testing.assert_allclose(oracle_mod.layer_norm(a["x"], a["gamma"], a["beta"], eps), ref,
                                   rtol=0, atol=1e-12)


def test_b2_zero_projection_leaves_the_residual(oracle_mod):
    # Wproj = 0 and bproj = 0: the attention branch is exactly zero and the block returns x
    shape, heads, window, shift = (1, 5, 9, 10, 32), 2, (4, 4, 4), (2, 2, 2)
    a = _block_inputs(shape, heads, window)
    a["Wproj"] = np.zeros_like(a["Wproj"])
    a["bproj"] = np.zeros_like(a["bproj"])
    out = _run_block(oracle_mod, a, window, shift, heads)
    assert np.array_equal(out, a["x"])


def test_b3_constant_tokens_closed_form(oracle_mod):
    # Tokens whose channels are all equal normalise to beta (zero variance), so with no
    # padding every token feeds the same key and value: whatever the mask and bias do,
    # each softmax row sums to 1 and the branch is (beta Wv + bv) Wproj + bproj.
    shape, heads, window, shift = (1, 4, 6, 6, 16), 2, (2, 3, 3), (1, 1, 1)
    a = _block_inputs(shape, heads, window)
    rng = np.random.default_rng(5)
    a["x"] = np.repeat(rng.normal(size=shape[:-1] + (1,)), shape[-1], axis=-1)
    C = shape[-1]
    v = a["beta"] @ a["Wqkv"][:, 2 * C:] + a["bqkv"][2 * C:]
    branch = v @ a["Wproj"] + a["bproj"]
    out = _run_block(oracle_mod, a, window, shift, heads)
    np.testing.assert_allclose(out, a["x"] + branch, rtol=0, atol=1e-12)


def test_b4_token_offset_invariance(oracle_mod):
    # layer norm removes a per-token offset c, so block(x + c) = block(x) + c
    shape, heads, window, shift = (1, 6, 9, 10, 32), 1, (4, 7, 7), (2, 3, 3)
    a = _block_inputs(shape, heads, window)
    c = np.random.default_rng(6).normal(scale=3.0, size=shape[:-1] + (1,))
    out0 = _run_block(oracle_mod, a, window, shift, heads)
    b = dict(a)
    b["x"] = a["x"] + c
    out1 = _run_block(oracle_mod, b, window, shift, heads)
    np.testing.assert_allclose(out1 - out0, np.broadcast_to(c, out0.shape), rtol=0, atol=1e-9)


def test_b5_padding_is_zero_after_the_norm(oracle_mod):
    # The norm comes before the padding: padded slots are zero tokens for the layer, not
    # the norm of zeros (beta). Built from the layer oracle on an explicitly padded input.
    shape, heads, window, shift = (1, 3, 5, 6, 16), 2, (2, 3, 3), (1, 1, 1)
    a = _block_inputs(shape, heads, window)
    y = oracle_mod.layer_norm(a["x"], a["gamma"], a["beta"])
    padded = np.zeros((1, 4, 6, 6, 16))
    padded[:, :3, :5, :6] = y
    full = oracle_mod.forward(padded, window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"], a["table"],
                              heads)
    out = _run_block(oracle_mod, a, window, shift, heads)
    np.testing.assert_allclose(out, a["x"] + full[:, :3, :5, :6], rtol=0, atol=1e-12)


# ---- MLP half of the block and the whole block --------------------------------------------------
def _mlp_params(C, hidden, seed):
    rng = np.random.default_rng(seed)
    return dict(gamma=1 + 0.1 * rng.normal(size=C), beta=0.1 * rng.normal(size=C),
                W1=rng.normal(size=(C, hidden)) / np.sqrt(C), b1=0.1 * rng.normal(size=hidden),
                W2=rng.normal(size=(hidden, C)) / np.sqrt(hidden), b2=0.1 * rng.normal(size=C))


def test_m1_gelu(oracle_mod):
    # against torch's exact GELU in float64, and the identity GELU(x) - GELU(-x) = x
    x = np.linspace(-6, 6, 241)
    ref = torch.nn.functional.gelu(torch.from_numpy(x)).numpy()
    np.testing.assert_allclose(oracle_mod.gelu(x), ref, rtol=0, atol=1e-14)
    np.testing.assert_allclose(oracle_mod.gelu(x) - oracle_mod.gelu(-x), x, rtol=0, atol=1e-14)
    assert oracle_mod.gelu(np.array([0.0]))[0] == 0.0


def test_m2_zero_second_layer_is_identity(oracle_mod):
    z = np.random.default_rng(1).normal(size=(2, 3, 4, 5, 16))
    p = _mlp_params(16, 64, 2)
    p["W2"] = np.zeros_like(p["W2"])
    p["b2"] = np.zeros_like(p["b2"])
    out = oracle_mod.mlp_half(z, p["gamma"], p["beta"], 1e-5, p["W1"], p["b1"], p["W2"], p["b2"])
    assert np.array_equal(out, z)


def test_m3_constant_tokens_closed_form(oracle_mod):
    # a token with equal channels normalises to beta: the branch is GELU(beta W1 + b1) W2 + b2
    rng = np.random.default_rng(3)
    z = np.repeat(rng.normal(size=(1, 2, 3, 4, 1)), 16, axis=-1)
    p = _mlp_params(16, 64, 4)
    branch = oracle_mod.gelu(p["beta"] @ p["W1"] + p["b1"]) @ p["W2"] + p["b2"]
    out = oracle_mod.mlp_half(z, p["gamma"], p["beta"], 1e-5, p["W1"], p["b1"], p["W2"], p["b2"])
    np.testing.assert_allclose(out, z + branch, rtol=0, atol=1e-12)


def test_m4_mlp_matches_torch_modules(oracle_mod):
    # the MLP half against torch's LayerNorm / Linear / GELU / Linear in float64
    z = np.random.default_rng(5).normal(size=(1, 2, 3, 4, 16)) * 2 + 0.5
    p = _mlp_params(16, 64, 6)
    t = torch.from_numpy
    y = torch.nn.functional.layer_norm(t(z), (16,), t(p["gamma"]), t(p["beta"]), 1e-5)
    h = torch.nn.functional.gelu(y @ t(p["W1"]) + t(p["b1"]))
    ref = (t(z) + h @ t(p["W2"]) + t(p["b2"])).numpy()
    out = oracle_mod.mlp_half(z, p["gamma"], p["beta"], 1e-5, p["W1"], p["b1"], p["W2"], p["b2"])
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_m5_whole_block_is_the_two_halves(oracle_mod):
    # eq. 1: z_hat = x + attention(LN(x)), z = z_hat + MLP(LN(z_hat)); checked through the
    # zero-projection special cases: with both branches' last weights and biases zero the
    # block is the identity, with only the MLP's zero it is the attention half
    shape, heads, window, shift = (1, 4, 6, 6, 16), 2, (2, 3, 3), (1, 1, 1)
    a = _block_inputs(shape, heads, window)
    attn = {k: a[k] for k in ("gamma", "beta", "Wqkv", "bqkv", "Wproj", "bproj", "table")}
    mlp = _mlp_params(16, 64, 7)
    mlp0 = dict(mlp, W2=np.zeros_like(mlp["W2"]), b2=np.zeros_like(mlp["b2"]))
    half = _run_block(oracle_mod, a, window, shift, heads)
    np.testing.assert_allclose(oracle_mod.block_full_forward(a["x"], attn, mlp0, window, shift, heads), half,
                               rtol=0, atol=0)
    attn0 = dict(attn, Wproj=np.zeros_like(attn["Wproj"]), bproj=np.zeros_like(attn["bproj"]))
    assert np.array_equal(oracle_mod.block_full_forward(a["x"], attn0, mlp0, window, shift, heads), a["x"])
    full = oracle_mod.block_full_forward(a["x"], attn, mlp, window, shift, heads)
    np.testing.assert_allclose(full, oracle_mod.mlp_half(half, mlp["gamma"], mlp["beta"], 1e-5, mlp["W1"],
                                                         mlp["b1"], mlp["W2"], mlp["b2"]), rtol=0, atol=0)


# ---- per-window entry points (used for sampled parity at full size) ----------------------------
def test_w1_forward_windows_match_the_layer(oracle_mod):
    # forward_windows returns, per listed window and real slot, the layer's output at the
    # slot's token (the pinned forward), and some value at padding slots
    shape, heads, window, shift = (2, 5, 9, 10, 16), 2, (4, 4, 4), (2, 1, 3)
    a = _inputs(shape, heads, window)
    full = _run(oracle_mod, a, window, shift, heads).reshape(-1, shape[-1])
    g = oracle_mod.geometry(*shape[1:4], window, shift)
    wins = [0, 3, g["nW"] - 1, g["nW"] + 5, 2 * g["nW"] - 1]
    y = oracle_mod.forward_windows(a["x"], window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"], a["table"],
                                   heads, wins)
    src, _, _ = oracle_mod.index_maps(shape[0], *shape[1:4], window, shift)
    N = g["N"]
    for k, w in enumerate(wins):
        s = src[w * N:(w + 1) * N]
        m = s >= 0
        np.testing.assert_allclose(y[k][m], full[s[m]], rtol=0, atol=1e-12)


def test_w2_block_forward_windows_match_the_block(oracle_mod):
    shape, heads, window, shift = (1, 5, 9, 10, 16), 2, (4, 4, 4), (2, 1, 3)
    a = _block_inputs(shape, heads, window)
    full = _run_block(oracle_mod, a, window, shift, heads).reshape(-1, shape[-1])
    g = oracle_mod.geometry(*shape[1:4], window, shift)
    wins = [0, 4, g["nW"] - 1]
    y = oracle_mod.block_forward_windows(a["x"], a["gamma"], a["beta"], 1e-5, window, shift, a["Wqkv"], a["bqkv"],
                                         a["Wproj"], a["bproj"], a["table"], heads, wins)
    src, _, _ = oracle_mod.index_maps(1, *shape[1:4], window, shift)
    N = g["N"]
    for k, w in enumerate(wins):
        s = src[w * N:(w + 1) * N]
        m = s >= 0
        np.testing.assert_allclose(y[k][m], full[s[m]], rtol=0, atol=1e-12)


# ---- patch merging ------------------------------------------------------------------------------
def test_pm1_gather_is_space_to_depth_up_to_a_channel_permutation(oracle_mod):
    # torch's pixel_unshuffle is the textbook 2x2 space-to-depth: output channel c*4 + dh*2 + dw
    # of (C, H, W) input holds x[c, 2i + dh, 2j + dw]. The oracle's gather must hold the same
    # values with channel (2 dw + dh) C + c.
    B, T, H, W, C = 2, 3, 6, 8, 5
    x = np.random.default_rng(3).standard_normal((B, T, H, W, C))
    g = oracle_mod.patch_merge_gather(x)
    xt = torch.from_numpy(x).permute(0, 1, 4, 2, 3).reshape(B * T, C, H, W)
    pu = torch.nn.functional.pixel_unshuffle(xt, 2).numpy()  # (BT, 4C, H/2, W/2)
    pu = pu.reshape(B, T, C, 2, 2, H // 2, W // 2)           # c, dh, dw
    ref = np.transpose(pu, (0, 1, 5, 6, 4, 3, 2)).reshape(B, T, H // 2, W // 2, 4 * C)  # dw, dh, c
    np.testing.assert_array_equal(g, ref)


def test_pm2_patch_merge_is_layer_norm_then_linear(oracle_mod):
    # LN over the 4C vector (torch's layer_norm) then x @ Wr (torch's linear), float64
    B, T, H, W, C = 1, 2, 4, 6, 8
    rng = np.random.default_rng(4)
    x = rng.standard_normal((B, T, H, W, C))
    gamma, beta = 1 + 0.1 * rng.standard_normal(4 * C), 0.1 * rng.standard_normal(4 * C)
    Wr, br = rng.standard_normal((4 * C, 2 * C)), rng.standard_normal(2 * C)
    y = oracle_mod.patch_merge(x, gamma, beta, 1e-5, Wr, br)
    xt = torch.from_numpy(x).permute(0, 1, 4, 2, 3).reshape(B * T, C, H, W)
    cat = torch.nn.functional.pixel_unshuffle(xt, 2).reshape(B, T, C, 2, 2, H // 2, W // 2)
    cat = cat.permute(0, 1, 5, 6, 4, 3, 2).reshape(B, T, H // 2, W // 2, 4 * C)
    z = torch.nn.functional.layer_norm(cat, (4 * C,), torch.from_numpy(gamma), torch.from_numpy(beta), 1e-5)
    ref = torch.nn.functional.linear(z, torch.from_numpy(Wr).T, torch.from_numpy(br)).numpy()
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)
    assert y.shape == (B, T, H // 2, W // 2, 2 * C)


def test_pm3_odd_extent_is_zero_padding(oracle_mod):
    # an odd H or W merges as if the input carried a zero row / column at the high end
    B, T, H, W, C = 1, 2, 5, 7, 4
    rng = np.random.default_rng(5)
    x = rng.standard_normal((B, T, H, W, C))
    xp = np.zeros((B, T, H + 1, W + 1, C))
    xp[:, :, :H, :W] = x
    np.testing.assert_array_equal(oracle_mod.patch_merge_gather(x), oracle_mod.patch_merge_gather(xp))
    assert oracle_mod.patch_merge_gather(x).shape == (B, T, 3, 4, 4 * C)


def test_pm4_no_temporal_merging_and_swin_t_shapes(oracle_mod):
    # The pages: Swin-T stage 1 (B, 56, 56, 96) merges to (B, 28, 28, 192) with no temporal
    # merging; a clip's frames stay separate (merging each frame alone gives the same result).
    B, T, H, W, C = 1, 3, 56, 56, 96
    rng = np.random.default_rng(6)
    x = rng.standard_normal((B, T, H, W, C)).astype(np.float32)
    gamma, beta = np.ones(4 * C), np.zeros(4 * C)
    Wr = rng.standard_normal((4 * C, 2 * C)) / np.sqrt(4 * C)
    y = oracle_mod.patch_merge(x, gamma, beta, 1e-5, Wr)
    assert y.shape == (B, T, 28, 28, 192)
    for t in range(T):
        yt = oracle_mod.patch_merge(x[:, t:t + 1], gamma, beta, 1e-5, Wr)
        np.testing.assert_allclose(y[:, t:t + 1], yt, rtol=0, atol=1e-12)
