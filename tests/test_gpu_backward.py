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
