"""GPU parity of e4m3 (fp8) window and full attention against the CPU fp64
oracle on the decoded inputs.  q, k, v are stored as OCP e4m3 bytes; each
tensor's values are its decoded e4m3 values times its descale factor, which is
what the oracle is given.  Q K^T runs on e4m3 tensor-core MMAs with fp32
accumulation (exact products), V is widened to bf16 exactly, and the P.V MMA,
the softmax and the bf16 output are those of the bf16 path, so the bounds are
the bf16 ones: max-abs <= 2e-2 and relative RMS <= 5e-3."""
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


def decoded(x, factor):
    return x.to(torch.float64).numpy() * (factor or 1.0)


CASES = [
    # shape, Hkv (0 = H), window, shift, descale (q, k, v), pad
    ((1, 1, 32, 32, 2, 128), 0, (1, 16, 16), (0, 8, 8), (0.0, 0.0, 0.0), False),
    ((2, 1, 32, 48, 3, 128), 0, (1, 16, 16), (0, 0, 8), (0.5, 0.25, 2.0), False),
    ((1, 14, 18, 32, 1, 128), 0, (7, 9, 16), (3, 4, 8), (0.0, 0.0, 0.0), False),  # video
    ((1, 1, 32, 32, 4, 128), 2, (1, 16, 16), (0, 8, 8), (0.0, 0.0, 0.0), False),  # grouped
    ((1, 1, 16, 16, 2, 128), 0, (1, 4, 8), (0, 2, 4), (0.0, 0.0, 0.0), False),
    ((1, 1, 20, 28, 2, 128), 0, (1, 16, 16), (0, 8, 8), (0.0, 0.0, 0.0), True),   # padded
]


@pytest.mark.parametrize("shape,Hkv,window,shift,descale,pad", CASES)
def test_e4m3_window_attention(basa, shape, Hkv, window, shift, descale, pad):
    B, T, Hg, Wg, H, d = shape
    hk = Hkv or H
    q, _, _ = make_qkv(shape, "e4m3", 501, 502, 503)
    _, k, v = make_qkv((B, T, Hg, Wg, hk, d), "e4m3", 501, 502, 503)
    flags = basa.BASA_FLAG_PAD_GRID if pad else 0
    out, lse = basa.window_attn(*(x.cuda() for x in (q, k, v)), window, shift, return_lse=True,
                                descale=descale, flags=flags)
    torch.cuda.synchronize()
    assert out.dtype == torch.bfloat16
    prm = oracle_params(shape, window, shift)
    prm.Hkv = Hkv
    prm.pad = pad
    ref, rl = oracle.window_attn(decoded(q, descale[0]), decoded(k, descale[1]),
                                 decoded(v, descale[2]), prm, want_lse=True)
    assert_close(out, ref, "bf16", f"{shape} {window} {shift} {descale}")
    assert float(np.abs(lse.double().cpu().numpy() - rl).max()) <= 2e-2
    assert basa.get_status() == 0


@pytest.mark.parametrize("shape", [(1, 1, 16, 40, 2, 128), (2, 1, 8, 20, 1, 128)])
def test_e4m3_full_attention(basa, shape):
    q, k, v = make_qkv(shape, "e4m3", 511, 512, 513)
    out = basa.full_attn(*(x.cuda() for x in (q, k, v)))
    torch.cuda.synchronize()
    B, T, Hg, Wg, H, d = shape
    ref = oracle.window_attn(decoded(q, 0), decoded(k, 0), decoded(v, 0),
                             oracle_params(shape, (T, Hg, Wg)))
    assert_close(out, ref, "bf16", f"full {shape}")


def test_e4m3_matches_bf16_path_on_the_same_values(basa):
    """e4m3 values are bf16 values: the e4m3 call and the bf16 call on the same
    (widened) inputs agree to the bf16 path's own rounding noise."""
    shape, window, shift = (1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8)
    q, k, v = (x.cuda() for x in make_qkv(shape, "e4m3", 521, 522, 523))
    a = basa.window_attn(q, k, v, window, shift)
    b = basa.window_attn(*(x.to(torch.bfloat16) for x in (q, k, v)), window, shift)
    torch.cuda.synchronize()
    assert float((a.float() - b.float()).abs().max()) <= 2e-2


def test_e4m3_refused_where_unsupported(basa):
    shape = (1, 1, 32, 32, 2, 128)
    q, k, v = (x.cuda() for x in make_qkv(shape, "e4m3", 531, 532, 533))
    with pytest.raises(basa.BasaError):
        basa.window_attn(q, k, v, (1, 16, 16), (0, 8, 8), pool=(1, 4, 4))
    q64, k64, v64 = (x.cuda() for x in make_qkv((1, 1, 32, 32, 2, 64), "e4m3", 1, 2, 3))
    with pytest.raises(basa.BasaError):
        basa.window_attn(q64, k64, v64, (1, 16, 16), (0, 8, 8))
