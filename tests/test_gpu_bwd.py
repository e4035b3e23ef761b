"""GPU parity of the window-attention backward (basa_window_attn_bwd) against
the CPU fp64 oracle's gradients.  fp32 (CUDA cores): max-abs <= 1e-5 on
gradients of unit scale.  bf16 (bf16 inputs, the bf16 forward's output and lse;
on the tensor cores fp32 logits and accumulators with P and dS rounded to bf16
as MMA operands, on CUDA cores fp32 throughout; gradients rounded once):
max-abs <= 2e-2 and relative RMS <= 5e-3, the forward's bf16 bounds.  The bf16
rounding of P and dS adds a relative error of at most 2^-9 per product term,
which leaves the relative RMS of a sum of many such terms near 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from basa_synth import make_qkv
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


CASES = [
    # shape, Hkv (0 = H), window, shift, dtype
    ((1, 1, 16, 16, 2, 64), 0, (1, 8, 8), (0, 4, 4), "f32"),
    ((2, 2, 8, 8, 2, 32), 0, (1, 4, 4), (1, 2, 2), "f32"),
    ((1, 1, 16, 16, 4, 128), 2, (1, 8, 8), (0, 4, 4), "f32"),
    ((1, 1, 32, 32, 2, 128), 0, (1, 16, 16), (0, 8, 8), "bf16"),
    ((1, 14, 18, 32, 1, 64), 0, (7, 9, 16), (3, 4, 8), "bf16"),
    ((1, 1, 32, 32, 4, 128), 2, (1, 16, 16), (0, 8, 8), "bf16"),
    ((2, 1, 32, 48, 3, 128), 0, (1, 16, 16), (0, 8, 0), "bf16"),
    ((1, 1, 32, 32, 2, 64), 0, (1, 8, 16), (0, 4, 8), "bf16"),
    ((1, 6, 10, 16, 2, 128), 0, (3, 5, 8), (1, 2, 0), "bf16"),
    ((1, 7, 9, 16, 8, 64), 2, (7, 9, 16), (0, 4, 8), "bf16"),
    ((1, 1, 16, 16, 2, 128), 0, (1, 4, 8), (0, 2, 4), "bf16"),
]


@pytest.mark.parametrize("shape,Hkv,window,shift,dtype", CASES)
def test_window_attention_backward(basa, shape, Hkv, window, shift, dtype):
    B, T, Hg, Wg, H, d = shape
    hk = Hkv or H
    q, _, _ = make_qkv(shape, dtype, 151, 152, 153)
    _, k, v = make_qkv((B, T, Hg, Wg, hk, d), dtype, 151, 152, 153)
    g, _, _ = make_qkv(shape, dtype, 154, 155, 156)
    dq_, dk_, dv_, dg = (x.cuda() for x in (q, k, v, g))
    out, lse = basa.window_attn(dq_, dk_, dv_, window, shift, return_lse=True)
    gq, gk, gv = basa.window_attn_bwd(dq_, dk_, dv_, out, dg, lse, window, shift)
    torch.cuda.synchronize()
    prm = oracle_params(shape, window, shift)
    prm.Hkv = Hkv
    f = oracle.as_f64
    rq, rk, rv = oracle.window_attn_bwd(f(q), f(k), f(v), f(g), prm)
    for got, ref, name in ((gq, rq, "dq"), (gk, rk, "dk"), (gv, rv, "dv")):
        assert_close(got, ref, dtype, f"{name} {shape} Hkv={Hkv}")


def test_backward_cuda_core_flag(basa):
    """BASA_FLAG_BWD_CUDA_CORES keeps the fp32 CUDA-core kernels reachable for bf16."""
    shape, window, shift = (1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8)
    q, k, v = make_qkv(shape, "bf16", 161, 162, 163)
    g, _, _ = make_qkv(shape, "bf16", 164, 165, 166)
    dq_, dk_, dv_, dg = (x.cuda() for x in (q, k, v, g))
    out, lse = basa.window_attn(dq_, dk_, dv_, window, shift, return_lse=True)
    grads = basa.window_attn_bwd(dq_, dk_, dv_, out, dg, lse, window, shift, flags=0x2)
    torch.cuda.synchronize()
    f = oracle.as_f64
    ref = oracle.window_attn_bwd(f(q), f(k), f(v), f(g), oracle_params(shape, window, shift))
    for got, r, name in zip(grads, ref, ("dq", "dk", "dv")):
        assert_close(got, r, "bf16", f"{name} CUDA cores")


def test_backward_flux1024_size(basa):
    """All 24 heads of the 64 x 64 FLUX 1024^2 latent grid with 16 x 16 windows
    shifted by 8: every gradient element against the oracle."""
    shape, window, shift = (1, 1, 64, 64, 24, 128), (1, 16, 16), (0, 8, 8)
    q, k, v = make_qkv(shape, "bf16", 171, 172, 173)
    g, _, _ = make_qkv(shape, "bf16", 174, 175, 176)
    dq_, dk_, dv_, dg = (x.cuda() for x in (q, k, v, g))
    out, lse = basa.window_attn(dq_, dk_, dv_, window, shift, return_lse=True)
    grads = basa.window_attn_bwd(dq_, dk_, dv_, out, dg, lse, window, shift)
    torch.cuda.synchronize()
    assert basa.get_status() == 0
    f = oracle.as_f64
    ref = oracle.window_attn_bwd(f(q), f(k), f(v), f(g), oracle_params(shape, window, shift))
    for got, r, name in zip(grads, ref, ("dq", "dk", "dv")):
        assert_close(got, r, "bf16", f"{name} flux1024")


POOLED = [
    # shape, Hkv (0 = H), window, shift, pool, dtype
    ((1, 1, 16, 16, 2, 64), 0, (1, 8, 8), (0, 4, 4), (1, 4, 4), "f32"),
    ((1, 2, 8, 8, 2, 32), 0, (1, 4, 4), (1, 2, 2), (2, 2, 2), "f32"),
    ((1, 1, 32, 32, 2, 128), 0, (1, 16, 16), (0, 8, 8), (1, 4, 4), "bf16"),
    ((1, 1, 32, 32, 4, 128), 2, (1, 16, 16), (0, 8, 8), (1, 4, 4), "bf16"),
    ((2, 1, 32, 32, 2, 64), 0, (1, 16, 16), (0, 8, 8), (1, 8, 8), "bf16"),
]


@pytest.mark.parametrize("shape,Hkv,window,shift,pool,dtype", POOLED)
def test_pooled_memory_backward(basa, shape, Hkv, window, shift, pool, dtype):
    """With K/V-pooled global memory: the pooled tokens' gradients reach every
    query's dq and flow back to k and v through the cell means."""
    B, T, Hg, Wg, H, d = shape
    hk = Hkv or H
    q, _, _ = make_qkv(shape, dtype, 181, 182, 183)
    _, k, v = make_qkv((B, T, Hg, Wg, hk, d), dtype, 181, 182, 183)
    g, _, _ = make_qkv(shape, dtype, 184, 185, 186)
    dq_, dk_, dv_, dg = (x.cuda() for x in (q, k, v, g))
    out, lse = basa.window_attn(dq_, dk_, dv_, window, shift, pool, return_lse=True)
    gq, gk, gv = basa.window_attn_bwd(dq_, dk_, dv_, out, dg, lse, window, shift, pool)
    torch.cuda.synchronize()
    assert basa.get_status() == 0
    prm = oracle_params(shape, window, shift, pool)
    prm.Hkv = Hkv
    f = oracle.as_f64
    rq, rk, rv = oracle.window_attn_bwd(f(q), f(k), f(v), f(g), prm)
    for got, ref, name in ((gq, rq, "dq"), (gk, rk, "dk"), (gv, rv, "dv")):
        assert_close(got, ref, dtype, f"{name} {shape} pool {pool} Hkv={Hkv}")


def test_backward_repeats_bit_for_bit_without_pooled_memory(basa):
    """Every gradient row of the window backward is owned by one unit and summed
    in a fixed order, so repeated calls agree bit for bit; with pooled memory the
    pooled gradients are summed with fp32 atomics in no fixed order, so repeats
    agree to within fp32 rounding of those sums (far below the bf16 output step)."""
    shape, window, shift = (1, 1, 32, 32, 4, 128), (1, 16, 16), (0, 8, 8)
    q, k, v = (x.cuda() for x in make_qkv(shape, "bf16", 191, 192, 193))
    g, _, _ = (x.cuda() for x in make_qkv(shape, "bf16", 194, 195, 196))
    for pool in ((0, 0, 0), (1, 4, 4)):
        out, lse = basa.window_attn(q, k, v, window, shift, pool, return_lse=True)
        a = basa.window_attn_bwd(q, k, v, out, g, lse, window, shift, pool)
        b = basa.window_attn_bwd(q, k, v, out, g, lse, window, shift, pool)
        torch.cuda.synchronize()
        for x, y in zip(a, b):
            if pool == (0, 0, 0):
                assert torch.equal(x, y)
            else:
                assert float((x.float() - y.float()).abs().max()) <= 2.0 ** -7 * float(x.float().abs().max())
    assert basa.get_status() == 0
