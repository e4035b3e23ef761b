"""GPU parity on grids that the window does not divide (BASA_FLAG_PAD_GRID)
against the CPU fp64 oracle with the same reading: each axis padded at its far
end to the next multiple of the window, the shift rolls the padded axis, and
padded positions are neither queries nor keys.  Bounds as everywhere: bf16
max-abs <= 2e-2 and relative RMS <= 5e-3, fp32 max-abs <= 1e-5."""
import numpy as np
import pytest
import torch

import oracle
from basa_synth import make_qkv, make_text_qkv
from gpu_util import assert_close, oracle_params

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def basa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_diffusion_basa_b200 import build
    build.build()
    import sparse_attention_diffusion_basa_b200 as m
    oracle.build_oracle()
    return m


def padded_params(shape, window, shift, pool=(0, 0, 0), Hkv=0):
    prm = oracle_params(shape, window, shift, pool)
    prm.pad = True
    prm.Hkv = Hkv
    return prm


FWD = [
    # shape, Hkv (0 = H), window, shift, pool, dtype
    ((1, 1, 48, 85, 2, 128), 0, (1, 16, 16), (0, 8, 8), (0, 0, 0), "bf16"),   # 1360 x 768 image
    ((1, 1, 20, 28, 2, 128), 0, (1, 16, 16), (0, 0, 0), (0, 0, 0), "bf16"),
    ((2, 1, 20, 28, 2, 64), 0, (1, 16, 16), (0, 8, 8), (0, 0, 0), "bf16"),
    ((1, 1, 5, 7, 2, 128), 0, (1, 16, 16), (0, 8, 8), (0, 0, 0), "bf16"),     # window > grid
    ((1, 13, 18, 32, 1, 128), 0, (7, 9, 16), (3, 4, 8), (0, 0, 0), "bf16"),   # padded t
    ((2, 5, 10, 16, 2, 64), 0, (3, 5, 8), (1, 2, 0), (0, 0, 0), "bf16"),      # padded t, 2 batches
    ((1, 1, 20, 28, 4, 128), 2, (1, 16, 16), (0, 8, 8), (1, 4, 4), "bf16"),   # pooled, grouped
    ((1, 1, 20, 28, 2, 64), 0, (1, 8, 8), (0, 4, 4), (0, 0, 0), "f32"),
    ((1, 3, 10, 9, 2, 32), 0, (2, 4, 4), (1, 2, 2), (1, 2, 3), "f32"),
]


@pytest.mark.parametrize("shape,Hkv,window,shift,pool,dtype", FWD)
def test_padded_window_attention(basa, shape, Hkv, window, shift, pool, dtype):
    B, T, Hg, Wg, H, d = shape
    hk = Hkv or H
    q, _, _ = make_qkv(shape, dtype, 401, 402, 403)
    _, k, v = make_qkv((B, T, Hg, Wg, hk, d), dtype, 401, 402, 403)
    out, lse = basa.window_attn(*(x.cuda() for x in (q, k, v)), window, shift, pool,
                                return_lse=True, flags=basa.BASA_FLAG_PAD_GRID)
    torch.cuda.synchronize()
    f = oracle.as_f64
    ref, rl = oracle.window_attn(f(q), f(k), f(v), padded_params(shape, window, shift, pool, Hkv),
                                 want_lse=True)
    assert_close(out, ref, dtype, f"{shape} {window} {shift}")
    tol = 1e-5 if dtype == "f32" else 2e-2
    assert float(np.abs(lse.double().cpu().numpy() - rl).max()) <= tol
    assert basa.get_status() == 0


def test_padding_changes_nothing_when_the_window_divides(basa):
    shape, window, shift = (1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8)
    q, k, v = (x.cuda() for x in make_qkv(shape, "bf16", 411, 412, 413))
    a = basa.window_attn(q, k, v, window, shift)
    b = basa.window_attn(q, k, v, window, shift, flags=basa.BASA_FLAG_PAD_GRID)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_grid_not_divided_without_the_flag_is_a_shape_error(basa):
    shape = (1, 1, 20, 28, 2, 128)
    q, k, v = (x.cuda() for x in make_qkv(shape, "bf16", 414, 415, 416))
    with pytest.raises(basa.BasaError):
        basa.window_attn(q, k, v, (1, 16, 16), (0, 8, 8))


BWD = [
    # shape, Hkv, window, shift, pool, dtype
    ((1, 1, 20, 28, 2, 128), 0, (1, 16, 16), (0, 8, 8), (0, 0, 0), "bf16"),
    ((1, 5, 10, 16, 2, 64), 0, (3, 5, 8), (1, 2, 0), (0, 0, 0), "bf16"),
    ((1, 1, 20, 28, 4, 64), 2, (1, 16, 16), (0, 8, 8), (1, 4, 4), "bf16"),
    ((1, 1, 10, 14, 2, 64), 0, (1, 8, 8), (0, 4, 4), (0, 0, 0), "f32"),
    ((1, 3, 10, 9, 2, 32), 0, (2, 4, 4), (1, 2, 2), (1, 2, 3), "f32"),
]


@pytest.mark.parametrize("shape,Hkv,window,shift,pool,dtype", BWD)
def test_padded_backward(basa, shape, Hkv, window, shift, pool, dtype):
    B, T, Hg, Wg, H, d = shape
    hk = Hkv or H
    q, _, _ = make_qkv(shape, dtype, 421, 422, 423)
    _, k, v = make_qkv((B, T, Hg, Wg, hk, d), dtype, 421, 422, 423)
    g, _, _ = make_qkv(shape, dtype, 424, 425, 426)
    dev = [x.cuda() for x in (q, k, v, g)]
    fl = basa.BASA_FLAG_PAD_GRID
    out, lse = basa.window_attn(*dev[:3], window, shift, pool, return_lse=True, flags=fl)
    grads = basa.window_attn_bwd(*dev[:3], out, dev[3], lse, window, shift, pool, flags=fl)
    torch.cuda.synchronize()
    f = oracle.as_f64
    refs = oracle.window_attn_bwd(f(q), f(k), f(v), f(g),
                                  padded_params(shape, window, shift, pool, Hkv))
    for got, ref, name in zip(grads, refs, ("dq", "dk", "dv")):
        assert_close(got, ref, dtype, f"{name} {shape}")
    assert basa.get_status() == 0


@pytest.mark.parametrize("shape,window,shift,L,dtype", [
    ((1, 1, 20, 28, 2, 128), (1, 16, 16), (0, 8, 8), 77, "bf16"),
    ((1, 1, 10, 14, 2, 64), (1, 8, 8), (0, 4, 4), 9, "f32"),
])
def test_padded_joint_forward_and_backward(basa, shape, window, shift, L, dtype):
    B, T, Hg, Wg, H, d = shape
    q, k, v = make_qkv(shape, dtype, 431, 432, 433)
    qt, kt, vt = make_text_qkv(B, L, H, d, dtype, 434, 435, 436)
    g, _, _ = make_qkv(shape, dtype, 437, 438, 439)
    gt, _, _ = make_text_qkv(B, L, H, d, dtype, 440, 441, 442)
    dev = [x.cuda() for x in (q, k, v, qt, kt, vt, g, gt)]
    fl = basa.BASA_FLAG_PAD_GRID
    out, out_t, lse, lse_t = basa.joint_attn(*dev[:6], window, shift, return_lse=True, flags=fl)
    grads = basa.joint_attn_bwd(*dev[:6], out, out_t, dev[6], dev[7], lse, lse_t, window, shift,
                                flags=fl)
    torch.cuda.synchronize()
    f = oracle.as_f64
    prm = padded_params(shape, window, shift)
    ref, ref_t = oracle.joint_attn(f(q), f(k), f(v), f(qt), f(kt), f(vt), prm)
    assert_close(out, ref, dtype, "image")
    assert_close(out_t, ref_t, dtype, "text")
    refs = oracle.joint_attn_bwd(f(q), f(k), f(v), f(qt), f(kt), f(vt), f(g), f(gt), prm)
    for got, r, name in zip(grads, refs, ("dq", "dk", "dv", "dqt", "dkt", "dvt")):
        assert_close(got, r, dtype, name)
    assert basa.get_status() == 0
