"""GPU parity of grouped-query attention (K/V with fewer heads than q; query
head h reads K/V head h / (H / Hkv)) against the CPU fp64 oracle, for window,
pooled, full and joint attention.  Same tolerances as the other parity tests."""
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


def _inputs(shape, Hkv, dtype, seed):
    B, T, Hg, Wg, H, d = shape
    q, _, _ = make_qkv(shape, dtype, seed, seed + 1, seed + 2)
    _, k, v = make_qkv((B, T, Hg, Wg, Hkv, d), dtype, seed, seed + 1, seed + 2)
    return q, k, v


def _prm(shape, window, shift=(0, 0, 0), pool=(0, 0, 0), Hkv=0):
    prm = oracle_params(shape, window, shift, pool)
    prm.Hkv = Hkv
    return prm


CASES = [
    # shape (q heads), Hkv, window, shift, pool, dtype
    ((1, 1, 32, 32, 4, 128), 2, (1, 16, 16), (0, 8, 8), (0, 0, 0), "bf16"),
    ((1, 1, 32, 32, 4, 128), 1, (1, 16, 16), (0, 8, 8), (1, 4, 4), "bf16"),
    ((1, 14, 18, 32, 4, 64), 2, (7, 9, 16), (3, 4, 8), (0, 0, 0), "bf16"),
    ((1, 1, 16, 16, 4, 64), 2, (1, 8, 8), (0, 4, 4), (1, 2, 2), "f32"),
]


@pytest.mark.parametrize("shape,Hkv,window,shift,pool,dtype", CASES)
def test_gqa_window(basa, shape, Hkv, window, shift, pool, dtype):
    q, k, v = _inputs(shape, Hkv, dtype, 101)
    out, lse = basa.window_attn(q.cuda(), k.cuda(), v.cuda(), window, shift, pool, return_lse=True)
    torch.cuda.synchronize()
    f = oracle.as_f64
    ref, rl = oracle.window_attn(f(q), f(k), f(v), _prm(shape, window, shift, pool, Hkv),
                                 want_lse=True)
    assert_close(out, ref, dtype, f"gqa {shape} Hkv={Hkv}")
    tol = 1e-5 if dtype == "f32" else 2e-2
    assert float(np.abs(lse.double().cpu().numpy() - rl).max()) <= tol
    assert basa.get_status() == 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gqa_full(basa, dtype):
    shape, Hkv = (1, 1, 16, 20, 4, 64), 2
    q, k, v = _inputs(shape, Hkv, dtype, 111)
    out = basa.full_attn(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    f = oracle.as_f64
    ref = oracle.full_attn(f(q), f(k), f(v), _prm(shape, (1, 16, 20), Hkv=Hkv))
    assert_close(out, ref, dtype, "gqa full")


def test_gqa_joint(basa):
    shape, Hkv, L = (1, 1, 32, 32, 4, 128), 2, 70
    B, T, Hg, Wg, H, d = shape
    q, k, v = _inputs(shape, Hkv, "bf16", 121)
    qt, _, _ = make_text_qkv(B, L, H, d, "bf16", 124, 125, 126)
    _, kt, vt = make_text_qkv(B, L, Hkv, d, "bf16", 124, 125, 126)
    out, out_t = basa.joint_attn(*(x.cuda() for x in (q, k, v, qt, kt, vt)), (1, 16, 16), (0, 8, 8))
    torch.cuda.synchronize()
    f = oracle.as_f64
    ref, ref_t = oracle.joint_attn(f(q), f(k), f(v), f(qt), f(kt), f(vt),
                                   _prm(shape, (1, 16, 16), (0, 8, 8), Hkv=Hkv))
    assert_close(out, ref, "bf16", "gqa joint image")
    assert_close(out_t, ref_t, "bf16", "gqa joint text")
