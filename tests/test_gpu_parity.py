"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle on the
same seeded inputs. Needs a B200."""

import numpy as np
import pytest
import torch

import oracle
from shifted_window_attention_sw_b200 import vswin
from shifted_window_attention_sw_b200.inputs import make_layer_inputs, workload_layer_inputs
from shifted_window_attention_sw_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu

# Tolerances. The headline gates are the layer's stated ones (bf16: max abs <= 2e-2,
# mean abs <= 2e-3; fp32: max abs <= 1e-4). At the baseline value scale those alone
# cannot see a dropped mask or bias (the output is ~4e-3 in magnitude), so every case
# also runs the sensitivity scale with scale-aware gates: relative L2 error and max
# error relative to the output's max. The bf16 path rounds q, k, v, P, the attention
# output and the result to bf16 (relative step 2^-8), which puts its relative L2 error
# near 3e-3; the gates leave about 3x room.
BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3
BF16_REL_L2, BF16_REL_MAX = 1e-2, 3e-2
F32_MAX_ABS, F32_REL_L2 = 1e-4, 1e-5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shifted_window_attention_sw_b200 import build

    build.build()
    oracle.build()
    vswin.lib()


def _oracle(a64, window, shift, heads, flags=0):
    return oracle.forward(a64["x"], window, shift, a64["Wqkv"], a64["bqkv"], a64["Wproj"], a64["bproj"],
                          a64["table"], heads, flags=flags)


def _gpu(inp, window, shift, heads, dtype):
    d = inp.to("cuda")
    fn = vswin.wmsa_forward if dtype == "bf16" else vswin.wmsa_forward_f32
    out = fn(d.x, window, shift, d.Wqkv, d.bqkv, d.Wproj, d.bproj, d.table, heads)
    assert vswin.poll_error() == vswin.OK, vswin.last_error()
    return out.double().cpu().numpy()


def _stats(out, ref):
    err = out - ref
    return {
        "max_abs": float(np.abs(err).max()),
        "mean_abs": float(np.abs(err).mean()),
        "rel_l2": float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30)),
        "rel_max": float(np.abs(err).max() / max(np.abs(ref).max(), 1e-30)),
    }


def _check_bf16(out, ref, sensitivity):
    s = _stats(out, ref)
    assert np.isfinite(out).all()
    assert s["max_abs"] <= BF16_MAX_ABS or sensitivity, s
    assert s["mean_abs"] <= BF16_MEAN_ABS or sensitivity, s
    assert s["rel_l2"] <= BF16_REL_L2, s
    assert s["rel_max"] <= BF16_REL_MAX, s
    return s


# ------------------------------------------------------------------ index maps (bit-exact)
@pytest.mark.parametrize(
    "B,T,H,W,window,shift",
    [
        (8, 16, 56, 56, (8, 7, 7), (4, 3, 3)),
        (8, 16, 56, 56, (8, 7, 7), (0, 0, 0)),
        (4, 12, 40, 40, (8, 7, 7), (4, 3, 3)),
        (32, 16, 14, 14, (8, 7, 7), (4, 3, 3)),
        (8, 16, 7, 7, (8, 7, 7), (4, 0, 0)),
        (1, 8, 14, 14, (8, 7, 7), (4, 3, 3)),
        (2, 5, 9, 10, (4, 4, 4), (2, 1, 3)),
        (1, 3, 7, 7, (8, 7, 7), (4, 3, 3)),    # every axis smaller than or equal to the window
        (2, 8, 14, 14, (8, 7, 7), (4, 3, 0)),
        (1, 1, 14, 21, (1, 7, 7), (0, 3, 3)),
    ],
)
def test_index_maps_bit_exact(B, T, H, W, window, shift):
    src_ref, reg_ref, bias_ref = oracle.index_maps(B, T, H, W, window, shift)
    src, reg, bias = vswin.index_maps(B, T, H, W, window, shift)
    torch.cuda.synchronize()
    assert np.array_equal(src.cpu().numpy(), src_ref)
    assert np.array_equal(reg.cpu().numpy(), reg_ref)
    assert np.array_equal(bias.cpu().numpy(), bias_ref)


# ------------------------------------------------------------------ fp32 path
@pytest.mark.parametrize("shift", [(4, 3, 3), (0, 0, 0), (0, 3, 3)])
@pytest.mark.parametrize("scale", ["baseline", "sensitivity"])
def test_f32_small_layer(shift, scale):
    wl = WORKLOADS["swin_t_s1_small_f32"]
    layer = wl.layers[0]
    inp = make_layer_inputs(layer.shape, layer.heads, layer.window, "f32", scale, seed=1000)
    ref = _oracle(inp.as_f64(), layer.window, shift, layer.heads)
    out = _gpu(inp, layer.window, shift, layer.heads, "f32")
    s = _stats(out, ref)
    assert s["max_abs"] <= F32_MAX_ABS, s
    assert s["rel_l2"] <= F32_REL_L2, s


@pytest.mark.parametrize(
    "shape,heads,window,shift",
    [
        ((1, 16, 14, 14, 64), 4, (16, 7, 7), (8, 3, 3)),   # temporal window 16 (N = 784), d = 16
        ((2, 5, 9, 10, 24), 2, (4, 4, 4), (2, 1, 3)),      # padding everywhere, d = 12
    ],
)
def test_f32_other_shapes(shape, heads, window, shift):
    inp = make_layer_inputs(shape, heads, window, "f32", "sensitivity", seed=4242)
    ref = _oracle(inp.as_f64(), window, shift, heads)
    out = _gpu(inp, window, shift, heads, "f32")
    s = _stats(out, ref)
    assert s["max_abs"] <= F32_MAX_ABS * max(1.0, np.abs(ref).max()), s
    assert s["rel_l2"] <= F32_REL_L2, s


# ------------------------------------------------------------------ bf16 path, whole layers
BF16_CASES = [
    # (shape, heads, window, shift)
    ((1, 8, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)),      # Swin-T width, 4 windows
    ((1, 8, 14, 14, 96), 3, (8, 7, 7), (0, 0, 0)),
    ((2, 16, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)),     # two temporal windows
    ((1, 12, 12, 12, 128), 4, (8, 7, 7), (4, 3, 3)),    # pads T, H, W
    ((1, 5, 9, 10, 32), 1, (8, 7, 7), (4, 3, 3)),       # every axis smaller than the window (not clamped)
    ((1, 16, 14, 14, 96), 3, (8, 7, 7), (4, 0, 0)),     # partial shifts
    ((1, 16, 14, 14, 96), 3, (8, 7, 7), (0, 3, 3)),
    ((1, 16, 14, 21, 64), 2, (8, 7, 7), (4, 3, 0)),
    ((1, 8, 14, 14, 384), 12, (8, 7, 7), (4, 3, 3)),    # Swin-T stage-3 width
    ((1, 8, 7, 7, 1024), 32, (8, 7, 7), (4, 0, 0)),     # Swin-B stage-4 width (K = 1024)
    ((1, 8, 7, 14, 544), 17, (8, 7, 7), (4, 0, 3)),     # 17 heads: projection BN = 32, tiled GEMMs
    ((2, 1, 14, 21, 64), 2, (1, 7, 7), (0, 3, 3)),      # 2D Swin special case
    ((1, 8, 14, 14, 64), 2, (4, 7, 7), (2, 3, 3)),      # temporal window 4
    ((2, 6, 14, 21, 64), 2, (2, 7, 7), (1, 3, 3)),      # temporal window 2 (one query tile per window)
    ((1, 20, 14, 14, 64), 2, (16, 7, 7), (8, 3, 3)),    # temporal window 16 (N = 784, one item buffer)
    ((1, 8, 8, 12, 64), 2, (4, 4, 4), (2, 2, 2)),
    ((2, 3, 4, 5, 32), 1, (1, 1, 1), (0, 0, 0)),        # one-token windows
    ((1, 4, 6, 6, 32), 1, (2, 2, 2), (1, 1, 1)),
]


@pytest.mark.parametrize("shape,heads,window,shift", BF16_CASES)
@pytest.mark.parametrize("scale", ["baseline", "sensitivity"])
def test_bf16_layer(shape, heads, window, shift, scale):
    inp = make_layer_inputs(shape, heads, window, "bf16", scale, seed=3000 + sum(shape))
    ref = _oracle(inp.as_f64(), window, shift, heads)
    out = _gpu(inp, window, shift, heads, "bf16")
    _check_bf16(out, ref, scale == "sensitivity")


@pytest.mark.parametrize("flag", [oracle.NO_MASK, oracle.POS_ROLL, oracle.NO_BIAS, oracle.ROLL_THEN_PAD])
def test_bf16_separates_plausible_slips(flag):
    # The GPU output must sit at least 10x closer to the oracle than to each mutant.
    shape, heads, window, shift = (1, 12, 12, 12, 64), 2, (8, 7, 7), (4, 3, 3)
    inp = make_layer_inputs(shape, heads, window, "bf16", "sensitivity", seed=99)
    a = inp.as_f64()
    ref = _oracle(a, window, shift, heads)
    mut = _oracle(a, window, shift, heads, flags=flag)
    out = _gpu(inp, window, shift, heads, "bf16")
    assert np.linalg.norm(out - ref) * 10 <= np.linalg.norm(out - mut)


@pytest.mark.parametrize("shape,heads,window,shift", [((1, 8, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)),
                                                     ((1, 4, 14, 14, 64), 2, (4, 7, 7), (2, 3, 3))])
def test_bf16_exact_softmax_rows(shape, heads, window, shift):
    # Every row through the kernel's exact two-pass recomputation (normally taken only
    # when the per-row reference is too loose): same parity gates as the fast path.
    inp = make_layer_inputs(shape, heads, window, "bf16", "sensitivity", seed=515)
    ref = _oracle(inp.as_f64(), window, shift, heads)
    vswin.set_exact_softmax(True)
    try:
        out = _gpu(inp, window, shift, heads, "bf16")
    finally:
        vswin.set_exact_softmax(False)
    _check_bf16(out, ref, True)


def test_bf16_large_logits():
    # Query/key magnitudes 6x the sensitivity scale: logits spread over tens of units,
    # the regime where the per-row reference is loosest.
    shape, heads, window, shift = (1, 8, 14, 14, 64), 2, (8, 7, 7), (4, 3, 3)
    inp = make_layer_inputs(shape, heads, window, "bf16", "sensitivity", seed=616)
    C = shape[-1]
    inp.Wqkv[:, :2 * C] = (inp.Wqkv[:, :2 * C].float() * 6.0).to(torch.bfloat16)
    ref = _oracle(inp.as_f64(), window, shift, heads)
    out = _gpu(inp, window, shift, heads, "bf16")
    assert np.isfinite(out).all()
    s = _stats(out, ref)
    assert s["rel_l2"] <= 5e-2, s  # peaked softmax: bf16 rounding of q and k moves the weights more


def test_bf16_deterministic():
    shape, heads, window, shift = (2, 16, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)
    d = make_layer_inputs(shape, heads, window, "bf16", "sensitivity", seed=7).to("cuda")
    o1 = vswin.wmsa_forward(d.x, window, shift, d.Wqkv, d.bqkv, d.Wproj, d.bproj, d.table, heads)
    o2 = vswin.wmsa_forward(d.x, window, shift, d.Wqkv, d.bqkv, d.Wproj, d.bproj, d.table, heads)
    assert vswin.poll_error() == vswin.OK
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("shape", [(1, 16, 14, 14, 96), (5, 8, 14, 21, 96), (3, 8, 7, 7, 96)])
def test_bf16_host_entry_matches_device_entry(shape):
    # the host entry pipelines groups of clips (5 clips: groups of 2, 2, 1; 3 clips: 1 each)
    heads, window, shift = 3, (8, 7, 7), (4, 3, 3)
    inp = make_layer_inputs(shape, heads, window, "bf16", "sensitivity", seed=8)
    d = inp.to("cuda")
    dev = vswin.wmsa_forward(d.x, window, shift, d.Wqkv, d.bqkv, d.Wproj, d.bproj, d.table, heads)
    xh = inp.x.clone().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    vswin.wmsa_forward_host(xh, window, shift, d.Wqkv, d.bqkv, d.Wproj, d.bproj, d.table, heads, oh)
    assert torch.equal(oh, dev.cpu())


# ------------------------------------------------------------------ full-size workloads, sampled
def _sample_windows(B, nW, nw):
    """First and last window of the batch, one window on the last row of each axis
    (where the shifted-window mask splits it) and one interior window."""
    def pos(i):
        return (i // (nw[1] * nw[2]), (i // nw[2]) % nw[1], i % nw[2])

    picks = {0, B * nW - 1, (B - 1) * nW + nW // 3}
    for a in range(3):
        cand = [i for i in range(nW) if pos(i)[a] == nw[a] - 1]
        picks.add((B // 2) * nW + cand[len(cand) // 2])
    return sorted(picks)


@pytest.mark.parametrize("wname", ["swin_t_s1_b8", "swin_t_s3_b32", "swin_b_pad_b4", "swin_b_stages_b8"])
def test_bf16_full_size_sampled(wname):
    wl = WORKLOADS[wname]
    for layer in wl.layers:
        inp = workload_layer_inputs(wl, layer, scale="sensitivity")
        out = _gpu(inp, layer.window, layer.shift, layer.heads, "bf16")
        g = oracle.geometry(layer.T, layer.H, layer.W, layer.window, layer.shift)
        wins = _sample_windows(layer.B, g["nW"], g["nw"])
        a = inp.as_f64()
        y = oracle.forward_windows(a["x"], layer.window, layer.shift, a["Wqkv"], a["bqkv"], a["Wproj"],
                                   a["bproj"], a["table"], layer.heads, wins)
        src, _, _ = oracle.index_maps(layer.B, layer.T, layer.H, layer.W, layer.window, layer.shift)
        flat = out.reshape(-1, layer.C)
        N = g["N"]
        got, exp = [], []
        for k, w in enumerate(wins):
            s = src[w * N:(w + 1) * N]
            m = s >= 0
            got.append(flat[s[m]])
            exp.append(y[k][m])
        _check_bf16(np.concatenate(got), np.concatenate(exp), True)
        assert np.isfinite(out).all()


def test_bf16_full_size_baseline_gates_headline():
    # The headline layer pair at the stated value scale, all outputs of the sampled windows.
    wl = WORKLOADS["swin_t_s1_b8"]
    for layer in wl.layers:
        inp = workload_layer_inputs(wl, layer, scale="baseline")
        out = _gpu(inp, layer.window, layer.shift, layer.heads, "bf16")
        g = oracle.geometry(layer.T, layer.H, layer.W, layer.window, layer.shift)
        wins = _sample_windows(layer.B, g["nW"], g["nw"])
        a = inp.as_f64()
        y = oracle.forward_windows(a["x"], layer.window, layer.shift, a["Wqkv"], a["bqkv"], a["Wproj"],
                                   a["bproj"], a["table"], layer.heads, wins)
        src, _, _ = oracle.index_maps(layer.B, layer.T, layer.H, layer.W, layer.window, layer.shift)
        flat = out.reshape(-1, layer.C)
        N = g["N"]
        for k, w in enumerate(wins):
            s = src[w * N:(w + 1) * N]
            m = s >= 0
            _check_bf16(flat[s[m]], y[k][m], False)


# ------------------------------------------------------------------ whole tensors: full size and multi-item
# The persistent kernels give each CTA several (window, head) items and several GEMM
# tiles only when a layer has more of them than the GPU has SMs. These cases compare
# every output element with the oracle on layers where every CTA runs several items
# (reused item buffers, barrier phases flipping across uses, a tile's epilogue deferred
# into the next item, alternating TMEM accumulators in the GEMMs), including the
# headline layers themselves.
@pytest.mark.parametrize("scale", ["baseline", "sensitivity"])
@pytest.mark.parametrize("k", [0, 1], ids=["wmsa", "swmsa"])
def test_bf16_headline_whole_tensor(k, scale):
    wl = WORKLOADS["swin_t_s1_b8"]
    layer = wl.layers[k]
    inp = workload_layer_inputs(wl, layer, scale=scale)
    out = _gpu(inp, layer.window, layer.shift, layer.heads, "bf16")
    ref = _oracle(inp.as_f64(), layer.window, layer.shift, layer.heads)
    _check_bf16(out, ref, scale == "sensitivity")


MULTI_ITEM_CASES = [
    # (shape, heads, window, shift): items = windows x heads, per CTA on 148 SMs
    ((8, 16, 28, 28, 96), 3, (8, 7, 7), (4, 3, 3)),    # 768 items (5.2 per CTA), 784 GEMM tiles
    ((8, 16, 28, 28, 96), 3, (8, 7, 7), (0, 0, 0)),
    ((8, 32, 28, 14, 128), 4, (16, 7, 7), (8, 3, 3)),  # N = 784, one item buffer: 512 items (3.5 per CTA)
    ((4, 16, 28, 28, 64), 2, (4, 7, 7), (2, 3, 3)),    # 512 items of N = 196
    ((8, 16, 32, 32, 64), 2, (4, 4, 4), (2, 2, 2)),    # generic kernel, 4096 items
]


@pytest.mark.parametrize("shape,heads,window,shift", MULTI_ITEM_CASES)
def test_bf16_multi_item_whole_tensor(shape, heads, window, shift):
    inp = make_layer_inputs(shape, heads, window, "bf16", "sensitivity", seed=7000 + sum(shape))
    ref = _oracle(inp.as_f64(), window, shift, heads)
    out = _gpu(inp, window, shift, heads, "bf16")
    _check_bf16(out, ref, True)


# ------------------------------------------------------------------ bounded waits
def test_timeout_path_reports_and_recovers():
    vswin.set_wait_limit_ns(20_000_000)  # 20 ms
    try:
        vswin.selftest_timeout()
        assert vswin.poll_error() == vswin.ERR_TIMEOUT
        assert vswin.poll_error() == vswin.OK  # the word is cleared by the poll
    finally:
        vswin.set_wait_limit_ns(1_000_000_000)
    # the context is still usable
    shape, heads, window, shift = (1, 8, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)
    inp = make_layer_inputs(shape, heads, window, "bf16", "sensitivity", seed=11)
    ref = _oracle(inp.as_f64(), window, shift, heads)
    _check_bf16(_gpu(inp, window, shift, heads, "bf16"), ref, True)
