"""The checked build (compiled with BASA_CHECKED): its kernels verify every TMA
box and every output index against their tensors.  On valid calls it must find
nothing (device status 0) and produce the same results as the normal build:
bit for bit where the kernels are deterministic, within fp32 rounding of the
pooled gradients' atomic sums for the backward with pooled memory."""
import pytest
import torch

from basa_synth import make_qkv, make_text_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_diffusion_basa_b200 import build
    normal, checked = build.build(), build.build(checked=True)
    import sparse_attention_diffusion_basa_b200 as m
    from sparse_attention_diffusion_basa_b200 import _lib
    return m, _lib, normal, checked


def run_both(libs, fn):
    """fn(module) with the normal library, then with the checked one."""
    m, _lib, normal, checked = libs
    saved = (_lib.LIB_PATH, _lib._lib)
    out = []
    try:
        for path in (normal, checked):
            _lib.LIB_PATH, _lib._lib = path, None
            res = fn(m)
            torch.cuda.synchronize()
            assert m.get_status() == 0, f"{path}: device status"
            out.append(res)
    finally:
        _lib.LIB_PATH, _lib._lib = saved
    return out


def _cuda(*xs):
    return [x.cuda() for x in xs]


@pytest.mark.parametrize("shape,window,shift,pool", [
    ((1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8), (1, 4, 4)),
    ((1, 14, 18, 32, 1, 64), (7, 9, 16), (3, 4, 8), (0, 0, 0)),   # TMA-store epilogue
    ((2, 6, 10, 16, 2, 128), (3, 5, 8), (1, 2, 0), (0, 0, 0)),
])
def test_checked_window_matches(libs, shape, window, shift, pool):
    q, k, v = _cuda(*make_qkv(shape, "bf16", 301, 302, 303))
    a, b = run_both(libs, lambda m: m.window_attn(q, k, v, window, shift, pool, return_lse=True))
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_checked_full_and_joint_match(libs):
    q, k, v = _cuda(*make_qkv((1, 1, 16, 20, 2, 128), "bf16", 311, 312, 313))
    a, b = run_both(libs, lambda m: m.full_attn(q, k, v))
    assert torch.equal(a, b)
    shape, L = (1, 1, 64, 64, 2, 128), 64       # the text pass splits its key range
    q, k, v = _cuda(*make_qkv(shape, "bf16", 321, 322, 323))
    qt, kt, vt = _cuda(*make_text_qkv(1, L, 2, 128, "bf16", 324, 325, 326))
    a, b = run_both(libs, lambda m: m.joint_attn(q, k, v, qt, kt, vt, (1, 16, 16), (0, 8, 8),
                                                 return_lse=True))
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_checked_backward_matches(libs):
    shape, window, shift, pool = (1, 1, 32, 32, 4, 128), (1, 16, 16), (0, 8, 8), (1, 4, 4)
    q, _, _ = make_qkv(shape, "bf16", 331, 332, 333)
    _, k, v = make_qkv((1, 1, 32, 32, 2, 128), "bf16", 331, 332, 333)
    g, _, _ = make_qkv(shape, "bf16", 334, 335, 336)
    q, k, v, g = _cuda(q, k, v, g)
    for pl in ((0, 0, 0), pool):
        def bwd(m):
            out, lse = m.window_attn(q, k, v, window, shift, pl, return_lse=True)
            return m.window_attn_bwd(q, k, v, out, g, lse, window, shift, pl)
        a, b = run_both(libs, bwd)
        for x, y in zip(a, b):
            if pl == (0, 0, 0):
                assert torch.equal(x, y)
            else:
                assert float((x.float() - y.float()).abs().max()) <= 2.0 ** -7 * float(x.float().abs().max())
