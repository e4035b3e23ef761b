"""GPU edge cases: degenerate windows, tiny and ragged token counts, and the
sizes the bf16 kernel refuses, each against the CPU fp64 oracle or the
documented error code."""
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


def test_fp32_single_token_windows_return_v(basa):
    """A 1x1x1 window holds only the query's own token: softmax weight 1, out = v."""
    shape = (1, 2, 4, 6, 2, 64)
    q, k, v = make_qkv(shape, "f32", 131, 132, 133)
    out = basa.window_attn(q.cuda(), k.cuda(), v.cuda(), (1, 1, 1), (1, 3, 5))
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), v)


def test_bf16_refuses_windows_below_its_tile_granularity(basa):
    from sparse_attention_diffusion_basa_b200 import BasaError
    q, k, v = (x.cuda() for x in make_qkv((1, 1, 8, 8, 2, 128), "bf16", 134, 135, 136))
    with pytest.raises(BasaError) as e:
        basa.window_attn(q, k, v, (1, 1, 1))
    assert e.value.code == 3  # BASA_ERR_UNSUPPORTED


@pytest.mark.parametrize("Wg", [1, 7, 129])
def test_bf16_full_attention_tiny_and_ragged(basa, Wg):
    shape = (2, 1, 1, Wg, 2, 128)
    q, k, v = make_qkv(shape, "bf16", 137, 138, 139)
    out, lse = basa.full_attn(q.cuda(), k.cuda(), v.cuda(), return_lse=True)
    torch.cuda.synchronize()
    ref, rl = oracle.full_attn(oracle.as_f64(q), oracle.as_f64(k), oracle.as_f64(v),
                               oracle_params(shape, (1, 1, Wg)), want_lse=True)
    assert_close(out, ref, "bf16", f"full N={Wg}")
    assert float(np.abs(lse.double().cpu().numpy() - rl).max()) <= 2e-2
    assert basa.get_status() == 0


def test_bf16_widest_window_row(basa):
    """ww = 128, the widest window row one tile takes, with a wrapped shift."""
    shape, window, shift = (1, 1, 4, 256, 2, 128), (1, 2, 128), (0, 1, 64)
    q, k, v = make_qkv(shape, "bf16", 140, 141, 142)
    out = basa.window_attn(q.cuda(), k.cuda(), v.cuda(), window, shift)
    torch.cuda.synchronize()
    ref = oracle.window_attn(oracle.as_f64(q), oracle.as_f64(k), oracle.as_f64(v),
                             oracle_params(shape, window, shift))
    assert_close(out, ref, "bf16", "widest window row")


def test_empty_batch_is_a_no_op(basa):
    q = torch.empty((0, 1, 16, 16, 2, 128), dtype=torch.bfloat16, device="cuda")
    out = basa.window_attn(q, q, q, (1, 16, 16), (0, 8, 8))
    torch.cuda.synchronize()
    assert out.shape == q.shape
