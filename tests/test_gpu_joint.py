"""GPU parity of joint text + image attention (basa_joint_attn) against the CPU
fp64 oracle: image queries attend to their shifted window plus every text token,
text queries attend to every token.  bf16: max-abs <= 2e-2 and relative RMS
<= 5e-3; fp32: max-abs <= 1e-5."""
import numpy as np
import pytest
import torch

import oracle
from basa_synth import WORKLOADS, make_qkv, make_text_qkv, text_inputs, workload_inputs
from gpu_util import assert_close, gather_rows, oracle_params, sample_queries

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
    # shape, window, shift, L, dtype
    ((1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8), 77, "bf16"),     # ragged text tile
    ((2, 1, 32, 48, 2, 128), (1, 16, 16), (0, 0, 8), 256, "bf16"),    # two full text tiles
    ((1, 1, 32, 32, 3, 64), (1, 16, 16), (0, 8, 8), 130, "bf16"),     # head dim 64
    ((1, 14, 18, 32, 1, 128), (7, 9, 16), (3, 4, 8), 300, "bf16"),    # video windows
    ((1, 1, 16, 20, 2, 128), (1, 16, 20), (0, 0, 0), 1, "bf16"),      # one text token
    ((1, 1, 16, 16, 2, 64), (1, 8, 8), (0, 4, 4), 45, "f32"),
    ((2, 2, 8, 8, 2, 32), (1, 4, 4), (1, 2, 2), 9, "f32"),
]


@pytest.mark.parametrize("shape,window,shift,L,dtype", CASES)
def test_joint_attention(basa, shape, window, shift, L, dtype):
    B, T, Hg, Wg, H, d = shape
    q, k, v = make_qkv(shape, dtype, 81, 82, 83)
    qt, kt, vt = make_text_qkv(B, L, H, d, dtype, 84, 85, 86)
    out, out_t, lse, lse_t = basa.joint_attn(*(x.cuda() for x in (q, k, v, qt, kt, vt)),
                                             window, shift, return_lse=True)
    torch.cuda.synchronize()
    f = oracle.as_f64
    ref, ref_t, rl, rl_t = oracle.joint_attn(f(q), f(k), f(v), f(qt), f(kt), f(vt),
                                             oracle_params(shape, window, shift), want_lse=True)
    assert_close(out, ref, dtype, f"image {shape} L={L}")
    assert_close(out_t, ref_t, dtype, f"text {shape} L={L}")
    tol = 1e-5 if dtype == "f32" else 2e-2
    assert float(np.abs(lse.double().cpu().numpy() - rl).max()) <= tol
    assert float(np.abs(lse_t.double().cpu().numpy() - rl_t).max()) <= tol
    assert basa.get_status() == 0


@pytest.mark.parametrize("shape,L", [((1, 1, 64, 64, 2, 128), 64),    # 33 key tiles in 7 splits
                                     ((2, 1, 32, 64, 1, 64), 200),    # head dim 64, ragged text
                                     ((1, 1, 64, 80, 3, 128), 300)])
def test_joint_text_pass_split_key_range(basa, shape, L):
    """Few text units: the text pass splits its key range over the SMs and
    merges the partials; both the split and the unsplit call match the oracle."""
    from sparse_attention_diffusion_basa_b200 import _lib
    import ctypes
    B, T, Hg, Wg, H, d = shape
    window, shift = (1, 16, 16), (0, 8, 8)
    prm = basa.make_params(shape, torch.bfloat16, window, shift)
    assert _lib.load().basa_joint_workspace_size(ctypes.byref(prm), L) > 0  # the pass splits
    q, k, v = make_qkv(shape, "bf16", 87, 88, 89)
    qt, kt, vt = make_text_qkv(B, L, H, d, "bf16", 94, 95, 96)
    args = [x.cuda() for x in (q, k, v, qt, kt, vt)]
    out, out_t, lse, lse_t = basa.joint_attn(*args, window, shift, return_lse=True)
    no_ws = torch.empty(0, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    f = oracle.as_f64
    ref, ref_t, rl, rl_t = oracle.joint_attn(f(q), f(k), f(v), f(qt), f(kt), f(vt),
                                             oracle_params(shape, window, shift), want_lse=True)
    assert_close(out, ref, "bf16", f"image {shape} L={L}")
    assert_close(out_t, ref_t, "bf16", f"text {shape} L={L} (split)")
    assert float(np.abs(lse_t.double().cpu().numpy() - rl_t).max()) <= 2e-2
    # the same call without a workspace runs the text pass unsplit
    raw = _lib.load()
    out_t2 = torch.empty_like(args[3])
    lse_t2 = torch.empty_like(lse_t)
    p = lambda x: ctypes.c_void_p(x.data_ptr())
    out2 = torch.empty_like(args[0])
    code = raw.basa_joint_attn(*(p(x) for x in args), L, p(out2), p(out_t2), None, p(lse_t2),
                               None, ctypes.byref(prm),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == 0
    torch.cuda.synchronize()
    assert_close(out_t2, ref_t, "bf16", f"text {shape} L={L} (unsplit)")
    assert float(np.abs(lse_t2.double().cpu().numpy() - rl_t).max()) <= 2e-2
    assert basa.get_status() == 0


def test_joint_without_text_is_window_attention(basa):
    shape, window, shift = (1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8)
    q, k, v = (x.cuda() for x in make_qkv(shape, "bf16", 91, 92, 93))
    empty = torch.empty((1, 0, 2, 128), dtype=torch.bfloat16, device="cuda")
    out, out_t = basa.joint_attn(q, k, v, empty, empty, empty, window, shift)
    ref = basa.window_attn(q, k, v, window, shift)
    torch.cuda.synchronize()
    assert torch.equal(out, ref) and out_t.numel() == 0


def test_joint_rejects_pooled_memory(basa):
    from sparse_attention_diffusion_basa_b200 import _lib
    import ctypes
    shape = (1, 1, 32, 32, 2, 128)
    q = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    t = torch.zeros((1, 4, 2, 128), dtype=torch.bfloat16, device="cuda")
    prm = basa.make_params(shape, torch.bfloat16, (1, 16, 16), (0, 8, 8), (1, 4, 4))
    p = lambda x: ctypes.c_void_p(x.data_ptr())
    code = _lib.load().basa_joint_attn(p(q), p(q), p(q), p(t), p(t), p(t), 4, p(q), p(t), None,
                                       None, None, ctypes.byref(prm), None)
    assert code == 3  # BASA_ERR_UNSUPPORTED


def test_flux1024_text512_sampled(basa):
    w = WORKLOADS["flux1024_text512"]
    q, k, v = workload_inputs(w, 0)
    qt, kt, vt = text_inputs(w, 0)
    shift = w.shifts[0]
    out, out_t, lse, lse_t = basa.joint_attn(*(x.cuda() for x in (q, k, v, qt, kt, vt)),
                                             w.window, shift, return_lse=True)
    torch.cuda.synchronize()
    assert basa.get_status() == 0
    sel = sample_queries(w.shape(), 256, 55)
    f = oracle.as_f64
    ref, ref_t, rl, rl_t = oracle.joint_attn(f(q), f(k), f(v), f(qt), f(kt), f(vt),
                                             oracle_params(w.shape(), w.window, shift),
                                             want_lse=True, select=sel)
    assert_close(gather_rows(out, sel), ref, "bf16", "flux1024_text512 image rows")
    assert_close(out_t, ref_t, "bf16", "flux1024_text512 text rows")
    got_lse = lse[torch.as_tensor(sel[:, 0]), torch.as_tensor(sel[:, 2]), torch.as_tensor(sel[:, 1])]
    assert float(np.abs(got_lse.double().cpu().numpy() - rl).max()) <= 2e-2
    assert float(np.abs(lse_t.double().cpu().numpy() - rl_t).max()) <= 2e-2
