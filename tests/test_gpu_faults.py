"""Failure paths on the GPU without a GPU fault.

* Host-side injection: an injected CUDA failure or scratch-allocation failure
  makes an entry call return its status before anything is launched, and the
  next call runs normally.
* The VSWIN_DEBUG_BOUNDS build (libvswin_debug.so): the same arithmetic as the
  ordinary build -- its outputs are bitwise equal -- plus index checks in the
  gathers and scatters. A row-table entry planted outside its extent sets the
  error word and the access is skipped. The planted token lies beyond the
  layer's tokens but inside the buffers this test allocates (they carry spare
  rows), so even an access the checks missed would stay in bounds.

The debug library runs in a child process (VSWIN_LIBRARY names it).
"""

import os
import subprocess
import sys

import pytest
import torch

from shifted_window_attention_sw_b200 import build as build_mod
from shifted_window_attention_sw_b200 import vswin
from shifted_window_attention_sw_b200.inputs import make_block_inputs, make_layer_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPE, HEADS, WINDOW, SHIFT = (1, 8, 14, 14, 96), 3, (8, 7, 7), (4, 3, 3)
PAD_SHAPE = (1, 6, 10, 12, 96)  # padding on every axis


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build_mod.build()


@pytest.mark.gpu
@pytest.mark.parametrize("kind, status", [(vswin.INJECT_CUDA, vswin.ERR_CUDA), (vswin.INJECT_ALLOC, vswin.ERR_NO_MEMORY)])
def test_injected_failure_launches_nothing(kind, status):
    _need_gpu()
    inp = make_layer_inputs(SHAPE, HEADS, WINDOW, "bf16", "baseline", seed=8100).to("cuda")
    args = (inp.x, WINDOW, SHIFT, inp.Wqkv, inp.bqkv, inp.Wproj, inp.bproj, inp.table, HEADS)
    ref = vswin.wmsa_forward(*args)
    torch.cuda.synchronize()
    before = vswin.launch_count()
    vswin.inject_failure(kind, 1)
    try:
        with pytest.raises(vswin.VswinError) as exc:
            vswin.wmsa_forward(*args)
        assert exc.value.status == status
        assert "injected" in vswin.last_error()
        assert vswin.launch_count() == before
    finally:
        vswin.inject_failure(kind, 0)
    again = vswin.wmsa_forward(*args)
    assert vswin.poll_error() == vswin.OK
    assert torch.equal(again, ref)


def _run_debug(code, tmp_path):
    lib = build_mod.build(debug_bounds=True)
    env = dict(os.environ, VSWIN_LIBRARY=lib, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600,
                       cwd=str(tmp_path))
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    return r.stdout


@pytest.mark.gpu
def test_debug_bounds_build_is_bitwise_equal(tmp_path):
    """Layer (shifted, and padded on every axis), fused block half and patch merge:
    the checked build gives the ordinary build's bits and raises no error."""
    _need_gpu()
    out = tmp_path / "debug.pt"
    code = f"""
import torch
from shifted_window_attention_sw_b200 import vswin
from shifted_window_attention_sw_b200.inputs import make_block_inputs, make_layer_inputs
assert vswin.debug_bounds_enabled()
res = []
for shape in ({SHAPE}, {PAD_SHAPE}):
    inp = make_layer_inputs(shape, {HEADS}, {WINDOW}, "bf16", "sensitivity", seed=8200).to("cuda")
    res.append(vswin.wmsa_forward(inp.x, {WINDOW}, {SHIFT}, inp.Wqkv, inp.bqkv, inp.Wproj, inp.bproj,
                                  inp.table, {HEADS}).cpu())
b = make_block_inputs({PAD_SHAPE}, {HEADS}, {WINDOW}, "bf16", "sensitivity", seed=8201).to("cuda")
L = b.layer
res.append(vswin.block_msa_forward(L.x, {WINDOW}, {SHIFT}, b.gamma, b.beta, 1e-5, L.Wqkv, L.bqkv, L.Wproj,
                                   L.bproj, L.table, {HEADS}).cpu())
C = L.x.shape[-1]
g = torch.Generator().manual_seed(8202)
Wr = (torch.randn(4 * C, 2 * C, generator=g) * 0.05).bfloat16().cuda()
res.append(vswin.patch_merge_forward(L.x, b.gamma.repeat(4), b.beta.repeat(4), 1e-5, Wr).cpu())
assert vswin.poll_error() == vswin.OK, vswin.last_error()
torch.save(res, {str(out)!r})
"""
    _run_debug(code, tmp_path)
    got = torch.load(out)
    ref = []
    for shape in (SHAPE, PAD_SHAPE):
        inp = make_layer_inputs(shape, HEADS, WINDOW, "bf16", "sensitivity", seed=8200).to("cuda")
        ref.append(vswin.wmsa_forward(inp.x, WINDOW, SHIFT, inp.Wqkv, inp.bqkv, inp.Wproj, inp.bproj,
                                      inp.table, HEADS).cpu())
    b = make_block_inputs(PAD_SHAPE, HEADS, WINDOW, "bf16", "sensitivity", seed=8201).to("cuda")
    L = b.layer
    ref.append(vswin.block_msa_forward(L.x, WINDOW, SHIFT, b.gamma, b.beta, 1e-5, L.Wqkv, L.bqkv, L.Wproj,
                                       L.bproj, L.table, HEADS).cpu())
    C = L.x.shape[-1]
    g = torch.Generator().manual_seed(8202)
    Wr = (torch.randn(4 * C, 2 * C, generator=g) * 0.05).bfloat16().cuda()
    ref.append(vswin.patch_merge_forward(L.x, b.gamma.repeat(4), b.beta.repeat(4), 1e-5, Wr).cpu())
    assert vswin.poll_error() == vswin.OK
    assert len(got) == len(ref)
    for k, (a, r) in enumerate(zip(got, ref)):
        assert torch.equal(a, r), k


@pytest.mark.gpu
def test_debug_bounds_catches_a_planted_row(tmp_path):
    """A row-table entry set beyond the layer's tokens: the gather
    and the scatter skip it, the poll reports VSWIN_ERR_BOUNDS, the spare rows
    of the buffers are untouched, and with the plant removed the next call is
    clean and equal to the ordinary build's output."""
    _need_gpu()
    out = tmp_path / "planted.pt"
    code = f"""
import torch
from shifted_window_attention_sw_b200 import vswin
from shifted_window_attention_sw_b200.inputs import make_layer_inputs
B, T, H, W, C = {SHAPE}
tokens = B * T * H * W
spare = 64
inp = make_layer_inputs({SHAPE}, {HEADS}, {WINDOW}, "bf16", "baseline", seed=8300).to("cuda")
xb = torch.full((tokens + spare, C), 7.0, dtype=torch.bfloat16, device="cuda")
xb[:tokens] = inp.x.reshape(tokens, C)
ob = torch.full((tokens + spare, C), -3.0, dtype=torch.bfloat16, device="cuda")
x = xb[:tokens].view(B, T, H, W, C)
o = ob[:tokens].view(B, T, H, W, C)
args = (x, {WINDOW}, {SHIFT}, inp.Wqkv, inp.bqkv, inp.Wproj, inp.bproj, inp.table, {HEADS})
vswin.debug_plant_row(5, tokens + 3)
vswin.wmsa_forward(*args, out=o)
st = vswin.poll_error()
spare_x = bool((xb[tokens:] == 7.0).all())
spare_o = bool((ob[tokens:] == -3.0).all())
vswin.debug_plant_row(-1, 0)
clean = vswin.wmsa_forward(*args)
st2 = vswin.poll_error()
torch.save(dict(st=st, st2=st2, spare_x=spare_x, spare_o=spare_o, clean=clean.cpu()), {str(out)!r})
"""
    _run_debug(code, tmp_path)
    r = torch.load(out)
    assert r["st"] == vswin.ERR_BOUNDS
    assert r["spare_x"] and r["spare_o"]
    assert r["st2"] == vswin.OK
    inp = make_layer_inputs(SHAPE, HEADS, WINDOW, "bf16", "baseline", seed=8300).to("cuda")
    ref = vswin.wmsa_forward(inp.x, WINDOW, SHIFT, inp.Wqkv, inp.bqkv, inp.Wproj, inp.bproj, inp.table, HEADS)
    assert torch.equal(r["clean"], ref.cpu())
