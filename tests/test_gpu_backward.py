"""GPU parity of the fp32 backward (vswin_wmsa_backward_f32) against the float64
gradient oracle (oracle/backward.py) on the same seeded inputs. Needs a B200."""

import numpy as np
import pytest
import torch

import oracle
from oracle import backward as oracle_backward
from shifted_window_attention_sw_b200 import vswin
from shifted_window_attention_sw_b200.inputs import make_layer_inputs

pytestmark = pytest.mark.gpu

NAMES = ("dx", "dWqkv", "dbqkv", "dWproj", "dbproj", "dtable")
# fp32 sums of a few hundred terms per product and atomics in the table and weight
# gradients: relative L2 error ~1e-6 expected; the gates leave two orders of room and
# sit three orders below what a wrong sign, index or dropped term produces.
REL_L2, REL_MAX = 1e-4, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shifted_window_attention_sw_b200 import build

    build.build()
    oracle.build()
    vswin.lib()


CASES = [
    # (shape, heads, window, shift)
    ((1, 3, 5, 6, 16), 2, (2, 3, 3), (1, 1, 1)),       # shifted, padding on two axes
    ((2, 2, 6, 6, 16), 2, (2, 3, 3), (0, 0, 0)),       # unshifted
    ((1, 8, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)),     # Swin-T width and window
    ((1, 5, 9, 10, 24), 2, (4, 4, 4), (2, 1, 3)),      # d = 12, padding everywhere
]


@pytest.mark.parametrize("shape,heads,window,shift", CASES)
def test_backward_f32(shape, heads, window, shift):
    inp = make_layer_inputs(shape, heads, window, "f32", "sensitivity", seed=7000 + sum(shape))
    dy = torch.randn(*shape, generator=torch.Generator().manual_seed(7100 + sum(shape)))
    a = inp.as_f64()
    ref = oracle_backward.backward(a["x"], window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"],
                                   a["table"], heads, dy.double().numpy())
    d = inp.to("cuda")
    got = vswin.wmsa_backward_f32(d.x, window, shift, d.Wqkv, d.bqkv, d.Wproj, d.bproj, d.table, heads,
                                  dy.to("cuda"))
    assert vswin.poll_error() == vswin.OK, vswin.last_error()
    for name, g, r in zip(NAMES, got, ref):
        g = g.double().cpu().numpy()
        assert g.shape == r.shape, name
        assert np.isfinite(g).all(), name
        err = g - r
        rel_l2 = np.linalg.norm(err) / max(np.linalg.norm(r), 1e-30)
        rel_max = np.abs(err).max() / max(np.abs(r).max(), 1e-30)
        assert rel_l2 <= REL_L2 and rel_max <= REL_MAX, (name, rel_l2, rel_max)


# bf16 backward (vswin_wmsa_backward, tcgen05). Inputs are bf16 values (the oracle
# gets the same values in float64). The path rounds q, k, v, O, dO, P, dS and dqkv to
# bf16 (relative 2^-9 = 2e-3 each, independent) and sums in fp32, so a few 1e-3 of
# relative error per gradient is expected (measured on these cases: relative L2
# <= 4.5e-3, relative max <= 7e-3). The gates, the forward's bf16 ones widened by half,
# leave about three times that and sit far below what a wrong sign, index, scale or
# dropped term gives (order 1).
BF16_REL_L2, BF16_REL_MAX = 1.5e-2, 3e-2
BF16_CASES = [
    # (shape, heads, window, shift)
    ((1, 8, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)),     # Swin-T width, shifted
    ((1, 8, 14, 14, 96), 3, (8, 7, 7), (0, 0, 0)),     # unshifted
    ((1, 12, 12, 12, 128), 4, (8, 7, 7), (4, 3, 3)),   # padding on every axis
    ((1, 4, 14, 14, 64), 2, (4, 7, 7), (2, 3, 3)),     # P = 4: two query tiles, two key blocks
    ((1, 2, 7, 14, 64), 2, (2, 7, 7), (1, 0, 3)),      # P = 2
    ((2, 1, 14, 21, 64), 2, (1, 7, 7), (0, 3, 3)),     # 2D Swin special case
]


@pytest.mark.parametrize("scale", ["baseline", "sensitivity"])
@pytest.mark.parametrize("shape,heads,window,shift", BF16_CASES)
def test_backward_bf16(shape, heads, window, shift, scale):
    inp = make_layer_inputs(shape, heads, window, "bf16", scale, seed=7200 + sum(shape))
    dy = torch.randn(*shape, generator=torch.Generator().manual_seed(7300 + sum(shape))).bfloat16()
    a = inp.as_f64()
    ref = oracle_backward.backward(a["x"], window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"],
                                   a["table"], heads, dy.double().numpy())
    d = inp.to("cuda")
    got = vswin.wmsa_backward(d.x, window, shift, d.Wqkv, d.bqkv, d.Wproj, d.bproj, d.table, heads,
                              dy.to("cuda"))
    assert vswin.poll_error() == vswin.OK, vswin.last_error()
    assert got[0].dtype == torch.bfloat16 and all(t.dtype == torch.float32 for t in got[1:])
    stats = {}
    for name, g, r in zip(NAMES, got, ref):
        g = g.double().cpu().numpy()
        assert g.shape == r.shape, name
        assert np.isfinite(g).all(), name
        err = g - r
        stats[name] = (np.linalg.norm(err) / max(np.linalg.norm(r), 1e-30),
                       np.abs(err).max() / max(np.abs(r).max(), 1e-30))
    print("bf16 backward", shape, window, shift, scale,
          {k: (float(f"{v[0]:.2e}"), float(f"{v[1]:.2e}")) for k, v in stats.items()})
    for name, (rel_l2, rel_max) in stats.items():
        assert rel_l2 <= BF16_REL_L2 and rel_max <= BF16_REL_MAX, (name, rel_l2, rel_max, stats)


def test_backward_bf16_chunked(tmp_path):
    """Windows in several chunks (a 1 MB scratch budget: three windows a chunk, the
    second chunk starting inside a clip) give the same gradients within the gates."""
    import subprocess
    import sys

    shape, heads, window, shift = (2, 8, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)
    out = tmp_path / "grads.pt"
    code = f"""
import torch
from shifted_window_attention_sw_b200 import vswin
from shifted_window_attention_sw_b200.inputs import make_layer_inputs
inp = make_layer_inputs({shape}, {heads}, {window}, "bf16", "sensitivity", seed=7400).to("cuda")
dy = torch.randn(*{shape}, generator=torch.Generator().manual_seed(7401)).bfloat16().cuda()
g = vswin.wmsa_backward(inp.x, {window}, {shift}, inp.Wqkv, inp.bqkv, inp.Wproj, inp.bproj, inp.table, {heads}, dy)
assert vswin.poll_error() == vswin.OK, vswin.last_error()
torch.save([t.cpu() for t in g], {str(out)!r})
"""
    env = dict(__import__("os").environ, VSWIN_CHUNK_MB="1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    got = torch.load(out)
    inp = make_layer_inputs(shape, heads, window, "bf16", "sensitivity", seed=7400)
    dy = torch.randn(*shape, generator=torch.Generator().manual_seed(7401)).bfloat16()
    a = inp.as_f64()
    ref = oracle_backward.backward(a["x"], window, shift, a["Wqkv"], a["bqkv"], a["Wproj"], a["bproj"],
                                   a["table"], heads, dy.double().numpy())
    for name, g, r in zip(NAMES, got, ref):
        g = g.double().numpy()
        err = g - r
        rel_l2 = np.linalg.norm(err) / max(np.linalg.norm(r), 1e-30)
        rel_max = np.abs(err).max() / max(np.abs(r).max(), 1e-30)
        assert rel_l2 <= BF16_REL_L2 and rel_max <= BF16_REL_MAX, (name, rel_l2, rel_max)
