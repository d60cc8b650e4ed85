"""The C ABI on the host: the library loads, exports every symbol the header
declares, and rejects bad arguments before launching anything. CPU only."""

import ctypes
import os
import re

import pytest

from shifted_window_attention_sw_b200 import build as build_mod
from shifted_window_attention_sw_b200 import vswin

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vswin.h")


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return vswin.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vswin_\w+)\s*\(", text)))


def test_header_declares_binding_exports():
    assert sorted(vswin.EXPORTS) == _declared()


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name
    assert vswin.version() >= 100


# fake device pointers: never dereferenced, because validation fails first
A16 = 1 << 20


def _call(fn, x=A16, B=1, T=8, H=14, W=14, C=96, heads=3, window=(8, 7, 7), shift=(4, 3, 3),
          Wqkv=A16 * 2, bqkv=A16 * 3, Wproj=A16 * 4, bproj=A16 * 5, table=A16 * 6, out=A16 * 64):
    w = (ctypes.c_int * 3)(*window) if window is not None else None
    s = (ctypes.c_int * 3)(*shift) if shift is not None else None
    p = lambda v: ctypes.c_void_p(v) if v else None  # noqa: E731
    return fn(p(x), B, T, H, W, C, heads, w, s, p(Wqkv), p(bqkv), p(Wproj), p(bproj), p(table), p(out), None)


@pytest.mark.parametrize("name", ["vswin_wmsa_forward", "vswin_wmsa_forward_f32"])
@pytest.mark.parametrize(
    "kw",
    [
        dict(B=0), dict(T=-1), dict(C=0), dict(heads=0),
        dict(C=96, heads=5),                      # C % heads != 0
        dict(shift=(8, 3, 3)),                    # shift >= window
        dict(shift=(-1, 0, 0)),
        dict(window=(0, 7, 7)),
        dict(window=None),
        dict(x=0), dict(out=0), dict(Wqkv=0), dict(bqkv=0), dict(Wproj=0), dict(bproj=0), dict(table=0),
        dict(x=A16 + 2),                          # misaligned
        dict(out=A16 + 8),                        # overlaps x
    ],
)
def test_invalid_arguments_launch_nothing(L, name, kw):
    before = vswin.launch_count()
    rc = _call(getattr(L, name), **kw)
    assert rc == vswin.ERR_INVALID_ARG, (rc, vswin.last_error())
    assert vswin.last_error()
    assert vswin.launch_count() == before


@pytest.mark.parametrize(
    "kw",
    [dict(C=128, heads=2),                          # head width 64
     dict(window=(3, 7, 7), shift=(1, 3, 3)),      # no kernel compiled for this window
     dict(window=(8, 8, 8), shift=(4, 4, 4))],     # N = 512, no kernel compiled for this window
)
def test_bf16_unsupported_shapes(L, kw):
    before = vswin.launch_count()
    rc = _call(L.vswin_wmsa_forward, **kw)
    assert rc == vswin.ERR_UNSUPPORTED, (rc, vswin.last_error())
    assert vswin.launch_count() == before


def _call_block(L, gamma=A16 * 7, beta=A16 * 8, eps=1e-5, **kw):
    # the block entry takes the layer's arguments with (gamma, beta, eps) after the shift
    captured = {}

    def fn(*args):
        captured["args"] = args
        return 0

    _call(fn, **kw)
    a = list(captured["args"])
    p = lambda v: ctypes.c_void_p(v) if v else None  # noqa: E731
    a[9:9] = [p(gamma), p(beta), ctypes.c_float(eps)]
    return L.vswin_block_msa_forward(*a)


@pytest.mark.parametrize(
    "kw",
    [
        dict(B=0), dict(C=96, heads=5), dict(shift=(8, 3, 3)), dict(window=None),
        dict(x=0), dict(out=0), dict(Wqkv=0), dict(table=0), dict(gamma=0), dict(beta=0),
        dict(gamma=A16 * 7 + 1),                  # misaligned
        dict(eps=-1e-5), dict(eps=float("nan")), dict(eps=float("inf")),
        dict(out=A16 + 64),                       # overlaps x without being x
    ],
)
def test_block_invalid_arguments_launch_nothing(L, kw):
    before = vswin.launch_count()
    rc = _call_block(L, **kw)
    assert rc == vswin.ERR_INVALID_ARG, (rc, vswin.last_error())
    assert vswin.last_error()
    assert vswin.launch_count() == before


@pytest.mark.parametrize("kw", [dict(C=128, heads=2), dict(window=(3, 7, 7), shift=(1, 3, 3))])
def test_block_unsupported_shapes(L, kw):
    # in place (out == x) passes the pointer checks; the shape is then refused
    before = vswin.launch_count()
    rc = _call_block(L, out=A16, **kw)
    assert rc == vswin.ERR_UNSUPPORTED, (rc, vswin.last_error())
    assert vswin.launch_count() == before


def test_index_maps_rejects_bad_window(L):
    w = (ctypes.c_int * 3)(8, 7, 7)
    s = (ctypes.c_int * 3)(8, 0, 0)
    rc = L.vswin_wmsa_index_maps(1, 8, 7, 7, w, s, None, None, None, None)
    assert rc == vswin.ERR_INVALID_ARG


@pytest.mark.parametrize(
    "dims,window,shift,ew,es",
    [
        ((16, 56, 56), (8, 7, 7), (4, 3, 3), (8, 7, 7), (4, 3, 3)),
        ((8, 14, 14), (8, 7, 7), (4, 3, 3), (8, 7, 7), (0, 3, 3)),   # T == P: window = 8, shift 0
        ((16, 7, 7), (8, 7, 7), (4, 3, 3), (8, 7, 7), (4, 0, 0)),    # Swin-B stage 4
        ((4, 5, 9), (8, 7, 7), (4, 3, 3), (4, 5, 7), (0, 0, 3)),
    ],
)
def test_clamp_window(L, dims, window, shift, ew, es):
    w, s = vswin.clamp_window(*dims, window, shift)
    assert w == ew and s == es


def _call_backward(L, dx=A16 * 9, dy=A16 * 10, **kw):
    # the backward entry takes the layer's arguments (without out) then dy and six gradients
    captured = {}

    def fn(*args):
        captured["args"] = args
        return 0

    _call(fn, **kw)
    a = list(captured["args"])
    p = lambda v: ctypes.c_void_p(v) if v else None  # noqa: E731
    grads = [p(dx), p(A16 * 11), p(A16 * 12), p(A16 * 13), p(A16 * 14), p(A16 * 15)]
    return L.vswin_wmsa_backward_f32(*(a[:14] + [p(dy)] + grads + [a[15]]))


@pytest.mark.parametrize(
    "kw",
    [dict(B=0), dict(window=None), dict(x=0), dict(dy=0), dict(dx=0), dict(Wqkv=0),
     dict(dx=A16 * 9 + 2),       # misaligned
     dict(dx=A16 + 64)],         # overlaps x
)
def test_backward_invalid_arguments_launch_nothing(L, kw):
    before = vswin.launch_count()
    rc = _call_backward(L, **kw)
    assert rc == vswin.ERR_INVALID_ARG, (rc, vswin.last_error())
    assert vswin.launch_count() == before


def test_binding_rejects_wrong_dtype_and_layout(L):
    # the Python binding checks dtypes, contiguity and shapes before calling the library
    import torch

    x = torch.zeros(1, 8, 14, 14, 96, dtype=torch.bfloat16)
    W = torch.zeros(96, 288, dtype=torch.bfloat16)
    b = torch.zeros(288, dtype=torch.bfloat16)
    Wp = torch.zeros(96, 96, dtype=torch.bfloat16)
    bp = torch.zeros(96, dtype=torch.bfloat16)
    t = torch.zeros(2535, 3, dtype=torch.bfloat16)
    before = vswin.launch_count()
    with pytest.raises(TypeError):
        vswin.wmsa_forward(x.float(), (8, 7, 7), (4, 3, 3), W, b, Wp, bp, t, 3)
    with pytest.raises(ValueError):
        vswin.wmsa_forward(x, (8, 7, 7), (4, 3, 3), W.t(), b, Wp, bp, t, 3)
    with pytest.raises(TypeError):
        vswin.block_msa_forward(x, (8, 7, 7), (4, 3, 3), bp.float(), bp, 1e-5, W, b, Wp, bp, t, 3)
    f = [a.float() for a in (x, W, b, Wp, bp, t)]
    with pytest.raises(ValueError):
        vswin.wmsa_backward_f32(*f[:1], (8, 7, 7), (4, 3, 3), *f[1:], 3, f[0][:, :4])
    assert vswin.launch_count() == before


@pytest.mark.parametrize("name", ["vswin_wmsa_forward", "vswin_wmsa_forward_f32", "vswin_wmsa_forward_noalloc"])
def test_layers_beyond_the_index_range_are_refused(L, name):
    # B * windows * N must stay below 2^31 (slot indices are 32-bit in the kernels)
    before = vswin.launch_count()
    rc = _call(getattr(L, name), B=1 << 20, T=16, H=56, W=56)
    assert rc == vswin.ERR_UNSUPPORTED, (rc, vswin.last_error())
    assert "2^31" in vswin.last_error()
    assert vswin.launch_count() == before


def test_block_and_backward_beyond_the_index_range_are_refused(L):
    before = vswin.launch_count()
    assert _call_block(L, B=1 << 20, T=16, H=56, W=56, out=A16) == vswin.ERR_UNSUPPORTED
    assert _call_backward(L, B=1 << 20, T=16, H=56, W=56) == vswin.ERR_UNSUPPORTED
    assert vswin.launch_count() == before


def _layer_tensors(dtype="bf16", C=96, heads=3, window=(8, 7, 7)):
    import torch

    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    rows = (2 * window[0] - 1) * (2 * window[1] - 1) * (2 * window[2] - 1)
    return dict(x=torch.zeros(1, 8, 14, 14, C, dtype=dt), Wqkv=torch.zeros(C, 3 * C, dtype=dt),
                bqkv=torch.zeros(3 * C, dtype=dt), Wproj=torch.zeros(C, C, dtype=dt), bproj=torch.zeros(C, dtype=dt),
                table=torch.zeros(rows, heads, dtype=dt))


@pytest.mark.parametrize("entry", ["wmsa_forward", "wmsa_forward_noalloc", "wmsa_forward_f32"])
def test_binding_rejects_host_tensors(L, entry):
    # The library reads raw device pointers: a CPU tensor must be refused by the binding,
    # before any call into the library.
    t = _layer_tensors("f32" if entry.endswith("f32") else "bf16")
    before = vswin.launch_count()
    with pytest.raises(ValueError, match="CUDA tensor"):
        getattr(vswin, entry)(t["x"], (8, 7, 7), (4, 3, 3), t["Wqkv"], t["bqkv"], t["Wproj"], t["bproj"],
                              t["table"], 3)
    assert vswin.launch_count() == before


def _fake_cuda(t):
    """A stand-in that passes the dtype / contiguity / device checks on a machine with no
    GPU (is_cuda and device report cuda:0) while keeping the real shape, so that the shape
    checks that follow can be exercised on the CPU."""
    import torch

    class Fake:
        def __init__(self, real):
            self.real = real
            self.shape = real.shape
            self.dtype = real.dtype
            self.is_cuda = True
            self.device = torch.device("cuda", 0)

        def is_contiguous(self):
            return True

        def dim(self):
            return self.real.dim()

    return Fake(t)


@pytest.mark.parametrize(
    "name,bad_shape",
    [("Wqkv", (96, 96)), ("Wqkv", (288, 96)), ("bqkv", (96,)), ("Wproj", (96, 48)), ("bproj", (288,)),
     ("table", (2535, 2)), ("table", (169, 3)), ("out", (1, 8, 14, 14, 48))],
)
def test_binding_rejects_wrong_shapes(L, name, bad_shape):
    # A short weight, table or output buffer would be read or written past its end by the
    # kernels: every shape the header fixes is checked before the library is called.
    import torch

    t = _layer_tensors()
    t["out"] = torch.zeros_like(t["x"])
    t[name] = torch.zeros(bad_shape, dtype=torch.bfloat16)
    f = {k: _fake_cuda(v) for k, v in t.items()}
    before = vswin.launch_count()
    with pytest.raises(ValueError, match="shape"):
        vswin.wmsa_forward(f["x"], (8, 7, 7), (4, 3, 3), f["Wqkv"], f["bqkv"], f["Wproj"], f["bproj"], f["table"],
                           3, out=f["out"])
    assert vswin.launch_count() == before


def test_binding_rejects_mixed_devices(L):
    import torch

    t = _layer_tensors()
    f = {k: _fake_cuda(v) for k, v in t.items()}
    f["table"].device = torch.device("cuda", 1)
    out = _fake_cuda(torch.zeros_like(t["x"]))
    with pytest.raises(ValueError, match="cuda:0"):
        vswin.wmsa_forward(f["x"], (8, 7, 7), (4, 3, 3), f["Wqkv"], f["bqkv"], f["Wproj"], f["bproj"], f["table"],
                           3, out=out)


def _call_mlp(L, x=A16, B=1, T=8, H=14, W=14, C=96, hidden=384, gamma=A16 * 7, beta=A16 * 8, eps=1e-5,
              W1=A16 * 2, b1=A16 * 3, W2=A16 * 4, b2=A16 * 5, out=A16 * 64):
    p = lambda v: ctypes.c_void_p(v) if v else None  # noqa: E731
    return L.vswin_mlp_forward(p(x), B, T, H, W, C, hidden, p(gamma), p(beta), ctypes.c_float(eps), p(W1), p(b1),
                               p(W2), p(b2), p(out), None)


@pytest.mark.parametrize(
    "kw",
    [dict(B=0), dict(C=0), dict(hidden=-1), dict(x=0), dict(out=0), dict(W1=0), dict(b1=0), dict(W2=0),
     dict(b2=0), dict(gamma=0), dict(beta=0),
     dict(W1=A16 * 2 + 8),          # not 16-byte aligned (TMA)
     dict(b1=A16 * 3 + 1),          # not 2-byte aligned
     dict(eps=-1.0), dict(eps=float("nan")),
     dict(out=A16 + 64)],           # overlaps x without being x
)
def test_mlp_invalid_arguments_launch_nothing(L, kw):
    before = vswin.launch_count()
    rc = _call_mlp(L, **kw)
    assert rc == vswin.ERR_INVALID_ARG, (rc, vswin.last_error())
    assert vswin.launch_count() == before


@pytest.mark.parametrize("kw", [dict(C=160, hidden=640), dict(C=48, hidden=192), dict(C=96, hidden=100),
                                dict(C=96, hidden=32 * 64), dict(B=1 << 20, T=16, H=56, W=56)])
def test_mlp_unsupported_shapes(L, kw):
    before = vswin.launch_count()
    rc = _call_mlp(L, out=A16, **kw)  # in place passes the pointer checks
    assert rc == vswin.ERR_UNSUPPORTED, (rc, vswin.last_error())
    assert vswin.launch_count() == before


def test_whole_block_checks_both_halves_before_launching(L):
    # a bad MLP argument must stop the call before the attention half is launched
    w = (ctypes.c_int * 3)(8, 7, 7)
    s = (ctypes.c_int * 3)(4, 3, 3)
    p = lambda k: ctypes.c_void_p(A16 * k)  # noqa: E731
    before = vswin.launch_count()
    for hidden, W1 in ((384, ctypes.c_void_p(A16 * 20 + 8)), (100, p(20))):  # misaligned W1; bad hidden
        rc = L.vswin_block_forward(p(1), 1, 8, 14, 14, 96, 3, w, s, p(2), p(3), p(4), p(5), p(6), p(7), p(8), p(9),
                                   p(10), hidden, W1, p(21), p(22), p(23), ctypes.c_float(1e-5), p(1), None)
        assert rc in (vswin.ERR_INVALID_ARG, vswin.ERR_UNSUPPORTED), (rc, vswin.last_error())
    assert vswin.launch_count() == before


def _call_merge(L, x=A16, B=1, T=8, H=14, W=14, C=96, gamma=A16 * 7, beta=A16 * 8, eps=1e-5, Wr=A16 * 2,
                br=A16 * 3, out=A16 * 64):
    p = lambda v: ctypes.c_void_p(v) if v else None  # noqa: E731
    return L.vswin_patch_merge_forward(p(x), B, T, H, W, C, p(gamma), p(beta), ctypes.c_float(eps), p(Wr), p(br),
                                       p(out), None)


@pytest.mark.parametrize(
    "kw",
    [dict(B=0), dict(W=-2), dict(C=0), dict(x=0), dict(out=0), dict(Wr=0), dict(gamma=0), dict(beta=0),
     dict(Wr=A16 * 2 + 4), dict(out=A16 * 64 + 2), dict(br=A16 * 3 + 1), dict(eps=float("inf")),
     dict(out=A16 + 128)],          # overlaps x
)
def test_patch_merge_invalid_arguments_launch_nothing(L, kw):
    before = vswin.launch_count()
    rc = _call_merge(L, **kw)
    assert rc == vswin.ERR_INVALID_ARG, (rc, vswin.last_error())
    assert vswin.launch_count() == before


def test_patch_merge_unsupported_width(L):
    before = vswin.launch_count()
    assert _call_merge(L, C=48) == vswin.ERR_UNSUPPORTED
    assert vswin.launch_count() == before


# ------------------------------------------------------------------ host-side fault injection
def _host_only():
    import torch

    return pytest.mark.skipif(torch.cuda.is_available(),
                              reason="calls with fake device pointers: only where no GPU can run them")


@_host_only()
def test_injected_cuda_failure_returns_before_the_device(L):
    """An injected CUDA failure makes the next entry calls return VSWIN_ERR_CUDA,
    naming the injection, before any device access; the count is exact."""
    before = vswin.launch_count()
    assert L.vswin_test_inject_failure(vswin.INJECT_CUDA, 2) == vswin.OK
    for name in ("vswin_wmsa_forward", "vswin_wmsa_forward_f32"):  # bf16 and fp32 entries
        assert _call(getattr(L, name)) == vswin.ERR_CUDA
        assert "injected" in vswin.last_error()
    # both consumed: the next call reaches the CUDA runtime, which has no device here
    assert _call(L.vswin_wmsa_forward) == vswin.ERR_CUDA
    assert "injected" not in vswin.last_error()
    assert vswin.launch_count() == before


@_host_only()
def test_injected_failure_cleared_by_count_zero(L):
    assert L.vswin_test_inject_failure(vswin.INJECT_CUDA, 5) == vswin.OK
    assert L.vswin_test_inject_failure(vswin.INJECT_CUDA, 0) == vswin.OK
    assert _call(L.vswin_wmsa_forward) == vswin.ERR_CUDA
    assert "injected" not in vswin.last_error()


def test_injection_rejects_bad_arguments(L):
    assert L.vswin_test_inject_failure(7, 1) == vswin.ERR_INVALID_ARG
    assert L.vswin_test_inject_failure(vswin.INJECT_ALLOC, -1) == vswin.ERR_INVALID_ARG
    assert L.vswin_test_inject_failure(vswin.INJECT_ALLOC, 0) == vswin.OK


def test_invalid_arguments_do_not_consume_an_injection(L):
    """Validation comes first: a rejected call leaves a pending injection in place."""
    assert L.vswin_test_inject_failure(vswin.INJECT_CUDA, 1) == vswin.OK
    assert _call(L.vswin_wmsa_forward, B=0) == vswin.ERR_INVALID_ARG
    assert L.vswin_test_inject_failure(vswin.INJECT_CUDA, 0) == vswin.OK


# ------------------------------------------------------------------ VSWIN_DEBUG_BOUNDS build
def test_plant_hook_needs_the_debug_build(L):
    assert L.vswin_debug_bounds_enabled() == 0
    assert L.vswin_debug_plant_row(3, 5) == vswin.ERR_UNSUPPORTED
    assert "VSWIN_DEBUG_BOUNDS" in vswin.last_error()


def test_debug_bounds_library_builds_and_exports_every_symbol():
    path = build_mod.build(debug_bounds=True)
    assert path == build_mod.LIB_DEBUG and os.path.exists(path)
    D = ctypes.CDLL(path)
    for name in _declared():
        assert hasattr(D, name), name
    D.vswin_debug_plant_row.argtypes = [ctypes.c_longlong, ctypes.c_int]
    assert D.vswin_debug_bounds_enabled() == 1
    assert D.vswin_debug_plant_row(3, 5) == vswin.OK
    assert D.vswin_debug_plant_row(-1, 0) == vswin.OK
