"""The no-allocation entry point (vswin_wmsa_forward_noalloc).

It serves callers that cannot allocate device memory while running the layer
(memory reserved up front, no device-wide synchronisation allowed, a foreign
allocator). Instead of stream-ordered scratch it streams windows through the
library's fixed 32 MiB device array, so its results must match the ordinary
entry point's, call after call, while the array keeps stale contents from the
previous call.

The two entry points run the same kernels on the same per-window inputs; only
the split of the windows into launch chunks differs, and no result depends on
which chunk (or which tile of a chunk) a window lands in: every output row is
one fixed-order accumulation over its own inputs. So the outputs must be
bitwise equal, not just close.

This file is named so that pytest collects it last.
"""

import ctypes

import pytest
import torch

from shifted_window_attention_sw_b200 import vswin
from shifted_window_attention_sw_b200.inputs import workload_layer_inputs
from shifted_window_attention_sw_b200.workloads import WORKLOADS

NOALLOC_BYTES = 32 << 20


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
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        torch_before = torch.cuda.memory_reserved()
        vswin.wmsa_forward_noalloc(d.x, layer.window, layer.shift, d.Wqkv, d.bqkv, d.Wproj, d.bproj, d.table,
                                   layer.heads, out=out)
        assert vswin.poll_error() == vswin.OK, vswin.last_error()
        # nothing was allocated: the device's free memory and torch's reservation are unchanged
        assert torch.cuda.mem_get_info()[0] == free_before
        assert torch.cuda.memory_reserved() == torch_before
        results.append((out, ref))
    for out, ref in results:
        assert torch.isfinite(out.float()).all()
        assert torch.equal(out, ref)


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
    msg = vswin.last_error()
    assert "scratch" in msg
    assert f"has {NOALLOC_BYTES} bytes" in msg  # the limit itself, 32 MiB
    needed = int(msg.split("needs ")[1].split(" bytes")[0])
    assert needed > NOALLOC_BYTES
    assert vswin.launch_count() == before
