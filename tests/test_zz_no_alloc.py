"""The no-allocation entry point (vswin_wmsa_forward_noalloc).

It serves callers that cannot allocate device memory while running the layer
(memory reserved up front, no device-wide synchronisation allowed, a foreign
allocator). Instead of stream-ordered scratch it streams windows through the
library's fixed 32 MiB device array, so its results must match the ordinary
entry point's, call after call, while the array keeps stale contents from the
previous call.

This file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from shifted_window_attention_sw_b200 import vswin
from shifted_window_attention_sw_b200.inputs import workload_layer_inputs
from shifted_window_attention_sw_b200.workloads import WORKLOADS

# The same bf16 gates as the parity tests: relative L2 error and max error
# relative to the output's max.
REL_L2, REL_MAX = 1e-2, 3e-2


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    assert np.isfinite(a).all()
    err = a - b
    rel_l2 = np.linalg.norm(err) / np.linalg.norm(b)
    rel_max = np.abs(err).max() / np.abs(b).max()
    assert rel_l2 <= REL_L2 and rel_max <= REL_MAX, (rel_l2, rel_max)


@pytest.mark.gpu
def test_noalloc_matches_allocating_entry_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from shifted_window_attention_sw_b200 import build

    build.build()
    wl = WORKLOADS["swin_t_s1_b8"]  # full size: the fixed array holds ~100 windows, so 10+ chunks
    results = []
    for layer in wl.layers:  # W-MSA, then SW-MSA: the second call starts on the first call's leftovers
        d = workload_layer_inputs(wl, layer, scale="sensitivity").to("cuda")
        ref = vswin.wmsa_forward(d.x, layer.window, layer.shift, d.Wqkv, d.bqkv, d.Wproj, d.bproj, d.table,
                                 layer.heads)
        out = torch.empty_like(d.x)
        vswin.wmsa_forward_noalloc(d.x, layer.window, layer.shift, d.Wqkv, d.bqkv, d.Wproj, d.bproj, d.table,
                                   layer.heads, out=out)
        assert vswin.poll_error() == vswin.OK, vswin.last_error()
        results.append((out, ref))
    for out, ref in results:
        _close(out, ref)


def test_noalloc_rejects_layers_beyond_its_scratch():
    # 400 heads of width 32: one window would need ~41 MB of scratch (> 32 MiB).
    # Validation fails before anything touches a device, so fake pointers are fine.
    L = vswin.lib()
    base = 1 << 24
    w = (ctypes.c_int * 3)(8, 7, 7)
    s = (ctypes.c_int * 3)(4, 3, 3)
    p = lambda k: ctypes.c_void_p(base * k)  # noqa: E731
    before = vswin.launch_count()
    rc = L.vswin_wmsa_forward_noalloc(p(1), 1, 8, 7, 7, 12800, 400, w, s, p(40), p(80), p(120), p(160), p(200),
                                      p(240), None)
    assert rc == vswin.ERR_UNSUPPORTED
    assert "32" in vswin.last_error() and "scratch" in vswin.last_error()
    assert vswin.launch_count() == before
