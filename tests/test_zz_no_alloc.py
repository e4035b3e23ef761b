"""basa_window_attn_noalloc: window attention with pooled global memory for
callers that cannot allocate device memory (for example an operator inside a
host framework that owns all device memory and gives it no workspace, or a
serving path that forbids cudaMalloc/cudaFree after start-up).

The entry point keeps the pooled K/V scratch in a fixed array inside the
library.  This test calls it through the C ABI and checks it against the
existing entry point (basa_window_attn with a caller workspace) within the
parity tolerances, on two calls in a row whose pooled scratch contents differ,
so stale scratch from the first call cannot leak into the second.

This file is collected last on purpose; it needs nothing from the other tests.
"""
import ctypes

import pytest
import torch

from basa_synth import make_qkv
from gpu_util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def basa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_diffusion_basa_b200 import build
    build.build()
    import sparse_attention_diffusion_basa_b200 as m
    return m


def _noalloc(basa, q, k, v, window, shift, pool):
    from sparse_attention_diffusion_basa_b200 import _lib
    lib = _lib.load()
    out = torch.empty_like(q)
    B, T, Hg, Wg, H, d = q.shape
    lse = torch.empty((B, H, T * Hg * Wg), dtype=torch.float32, device=q.device)
    prm = basa.make_params(q.shape, q.dtype, window, shift, pool)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = lib.basa_window_attn_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                        ctypes.c_void_p(lse.data_ptr()), ctypes.byref(prm), stream)
    assert code == 0, _lib.STATUS_NAMES.get(code, code)
    return out, lse


CALLS = [
    # (shape, dtype, window, shift, pool, seed): two different problems in a row
    ((1, 1, 32, 32, 2, 128), "bf16", (1, 16, 16), (0, 8, 8), (1, 4, 4), 81),
    ((2, 1, 32, 48, 2, 128), "bf16", (1, 16, 16), (0, 8, 0), (1, 2, 2), 91),
]


@pytest.mark.parametrize("order", [(0, 1), (1, 0)])
def test_noalloc_matches_window_attn_on_two_calls(basa, order):
    for idx in order:
        shape, dtype, window, shift, pool, seed = CALLS[idx]
        q, k, v = (x.cuda() for x in make_qkv(shape, dtype, seed, seed + 1, seed + 2))
        got, got_lse = _noalloc(basa, q, k, v, window, shift, pool)
        want, want_lse = basa.window_attn(q, k, v, window, shift, pool, return_lse=True)
        torch.cuda.synchronize()
        assert_close(got, want.double().cpu().numpy(), dtype, f"noalloc call {idx}")
        assert float((got_lse - want_lse).abs().max()) <= 2e-2
    assert basa.get_status() == 0


def test_noalloc_fp32_matches_window_attn(basa):
    shape, window, shift, pool = (1, 2, 12, 10, 2, 64), (2, 6, 5), (1, 4, 2), (1, 2, 5)
    q, k, v = (x.cuda() for x in make_qkv(shape, "f32", 95, 96, 97))
    for _ in range(2):
        got, _ = _noalloc(basa, q, k, v, window, shift, pool)
        want = basa.window_attn(q, k, v, window, shift, pool)
        torch.cuda.synchronize()
        assert_close(got, want.double().cpu().numpy(), "f32", "noalloc fp32")
