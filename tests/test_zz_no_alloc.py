"""basa_window_attn_noalloc: window attention with pooled global memory for
callers that cannot allocate device memory (for example an operator inside a
host framework that owns all device memory and gives it no workspace, or a
serving path that forbids cudaMalloc/cudaFree after start-up).

The entry point keeps the pooled K/V scratch in a fixed array inside the
library.  It runs the same kernels as basa_window_attn on the same inputs, so
this test calls it through the C ABI and requires the same bits as the
existing entry point (basa_window_attn with a caller workspace), on two calls
in a row whose pooled scratch contents differ, so stale scratch from the first
call cannot leak into the second.  One case is also checked against the CPU
fp64 oracle at the parity tolerances, and the cases cover grouped K/V heads
(scratch laid out over the K/V heads) and a call without pooling (no scratch).

This file is collected last on purpose; it needs nothing from the other tests.
"""
import ctypes

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


def _noalloc(basa, q, k, v, window, shift, pool):
    from sparse_attention_diffusion_basa_b200 import _lib
    lib = _lib.load()
    out = torch.empty_like(q)
    B, T, Hg, Wg, H, d = q.shape
    Hkv = k.shape[-2]
    lse = torch.empty((B, H, T * Hg * Wg), dtype=torch.float32, device=q.device)
    prm = basa.make_params(q.shape, q.dtype, window, shift, pool, hkv=0 if Hkv == H else Hkv)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = lib.basa_window_attn_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                        ctypes.c_void_p(lse.data_ptr()), ctypes.byref(prm), stream)
    assert code == 0, _lib.STATUS_NAMES.get(code, code)
    return out, lse


def _inputs(shape, Hkv, dtype, seed):
    B, T, Hg, Wg, H, d = shape
    q, k, v = make_qkv(shape, dtype, seed, seed + 1, seed + 2)
    if Hkv and Hkv != H:
        _, k, v = make_qkv((B, T, Hg, Wg, Hkv, d), dtype, seed, seed + 1, seed + 2)
    return q.cuda(), k.cuda(), v.cuda()


CALLS = [
    # (shape, Hkv, dtype, window, shift, pool, seed): different problems in a row
    ((1, 1, 32, 32, 2, 128), 0, "bf16", (1, 16, 16), (0, 8, 8), (1, 4, 4), 81),
    ((2, 1, 32, 48, 2, 128), 0, "bf16", (1, 16, 16), (0, 8, 0), (1, 2, 2), 91),
    ((1, 1, 32, 32, 4, 128), 2, "bf16", (1, 16, 16), (0, 8, 8), (1, 4, 4), 85),
    ((1, 1, 32, 32, 2, 128), 0, "bf16", (1, 16, 16), (0, 8, 8), (0, 0, 0), 87),
]


@pytest.mark.parametrize("order", [(0, 1, 2, 3), (3, 2, 1, 0)])
def test_noalloc_matches_window_attn_on_calls_in_a_row(basa, order):
    for idx in order:
        shape, Hkv, dtype, window, shift, pool, seed = CALLS[idx]
        q, k, v = _inputs(shape, Hkv, dtype, seed)
        got, got_lse = _noalloc(basa, q, k, v, window, shift, pool)
        want, want_lse = basa.window_attn(q, k, v, window, shift, pool, return_lse=True)
        torch.cuda.synchronize()
        assert torch.equal(got, want), f"noalloc call {idx}: output bits differ"
        assert torch.equal(got_lse, want_lse), f"noalloc call {idx}: lse bits differ"
    assert basa.get_status() == 0


def test_noalloc_against_the_oracle(basa):
    shape, Hkv, dtype, window, shift, pool, seed = CALLS[2]
    q, k, v = _inputs(shape, Hkv, dtype, seed)
    for _ in range(2):
        got, got_lse = _noalloc(basa, q, k, v, window, shift, pool)
        torch.cuda.synchronize()
        prm = oracle_params(shape, window, shift, pool)
        prm.Hkv = Hkv
        f = oracle.as_f64
        ref, ref_lse = oracle.window_attn(f(q), f(k), f(v), prm, want_lse=True)
        assert_close(got, ref, dtype, "noalloc vs oracle")
        assert float(np.abs(got_lse.double().cpu().numpy() - ref_lse).max()) <= 2e-2
    assert basa.get_status() == 0


def test_noalloc_fp32_matches_window_attn(basa):
    shape, window, shift, pool = (1, 2, 12, 10, 2, 64), (2, 6, 5), (1, 4, 2), (1, 2, 5)
    q, k, v = (x.cuda() for x in make_qkv(shape, "f32", 95, 96, 97))
    for _ in range(2):
        got, _ = _noalloc(basa, q, k, v, window, shift, pool)
        want = basa.window_attn(q, k, v, window, shift, pool)
        torch.cuda.synchronize()
        assert torch.equal(got, want), "noalloc fp32: output bits differ"
        prm = oracle_params(shape, window, shift, pool)
        ref = oracle.window_attn(oracle.as_f64(q), oracle.as_f64(k), oracle.as_f64(v), prm)
        assert_close(got, ref, "f32", "noalloc fp32 vs oracle")
