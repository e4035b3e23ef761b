"""GPU parity of the joint text + image backward (basa_joint_attn_bwd) against
the CPU fp64 oracle's gradients: image queries see their shifted window and the
L text keys, text queries see every image and text key, and the text keys
collect gradient from every query.  bf16 runs on the tensor cores (P and dS
rounded to bf16 as MMA operands, fp32 accumulation, the text keys' sums in
fp32), fp32 on CUDA cores; gradients rounded once.  The bounds are the
forward's: fp32 max-abs <= 1e-5, bf16 max-abs <= 2e-2 and relative RMS
<= 5e-3."""
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


CASES = [
    # shape, Hkv (0 = H), window, shift, L, dtype
    ((1, 1, 16, 16, 2, 64), 0, (1, 8, 8), (0, 4, 4), 45, "f32"),
    ((2, 2, 8, 8, 2, 32), 0, (1, 4, 4), (1, 2, 2), 9, "f32"),
    ((1, 1, 16, 16, 4, 64), 2, (1, 8, 8), (0, 4, 4), 33, "f32"),     # text keys shared by 2 heads
    ((1, 1, 32, 32, 2, 128), 0, (1, 16, 16), (0, 8, 8), 77, "bf16"),
    ((1, 14, 18, 32, 1, 64), 0, (7, 9, 16), (3, 4, 8), 130, "bf16"),  # video windows
    ((2, 1, 32, 48, 4, 128), 2, (1, 16, 16), (0, 0, 8), 256, "bf16"),
    ((1, 1, 16, 20, 2, 128), 0, (1, 16, 20), (0, 0, 0), 1, "bf16"),   # one text token
]


def run_case(basa, shape, Hkv, window, shift, L, dtype, seed=171, flags=0):
    B, T, Hg, Wg, H, d = shape
    hk = Hkv or H
    q, _, _ = make_qkv(shape, dtype, seed, seed + 1, seed + 2)
    _, k, v = make_qkv((B, T, Hg, Wg, hk, d), dtype, seed, seed + 1, seed + 2)
    g, _, _ = make_qkv(shape, dtype, seed + 3, seed + 4, seed + 5)
    qt, _, _ = make_text_qkv(B, L, H, d, dtype, seed + 6, seed + 7, seed + 8)
    _, kt, vt = make_text_qkv(B, L, hk, d, dtype, seed + 6, seed + 7, seed + 8)
    gt, _, _ = make_text_qkv(B, L, H, d, dtype, seed + 9, seed + 10, seed + 11)
    dev = [x.cuda() for x in (q, k, v, qt, kt, vt, g, gt)]
    out, out_t, lse, lse_t = basa.joint_attn(*dev[:6], window, shift, return_lse=True)
    grads = basa.joint_attn_bwd(*dev[:6], out, out_t, dev[6], dev[7], lse, lse_t, window, shift,
                                flags=flags)
    torch.cuda.synchronize()
    prm = oracle_params(shape, window, shift)
    prm.Hkv = Hkv
    f = oracle.as_f64
    refs = oracle.joint_attn_bwd(f(q), f(k), f(v), f(qt), f(kt), f(vt), f(g), f(gt), prm)
    return grads, refs


@pytest.mark.parametrize("shape,Hkv,window,shift,L,dtype", CASES)
def test_joint_attention_backward(basa, shape, Hkv, window, shift, L, dtype):
    grads, refs = run_case(basa, shape, Hkv, window, shift, L, dtype)
    for got, ref, name in zip(grads, refs, ("dq", "dk", "dv", "dqt", "dkt", "dvt")):
        assert_close(got, ref, dtype, f"{name} {shape} Hkv={Hkv} L={L}")
    assert basa.get_status() == 0


def test_joint_backward_without_text_is_the_window_backward(basa):
    """L = 0: the call is the window backward (text gradients are empty)."""
    shape, window, shift = (1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8)
    q, k, v = (x.cuda() for x in make_qkv(shape, "bf16", 181, 182, 183))
    g, _, _ = (x.cuda() for x in make_qkv(shape, "bf16", 184, 185, 186))
    e = torch.empty(1, 0, 2, 128, dtype=torch.bfloat16, device="cuda")
    out, _, lse, lse_t = basa.joint_attn(q, k, v, e, e, e, window, shift, return_lse=True)
    j = basa.joint_attn_bwd(q, k, v, e, e, e, out, e, g, e, lse, lse_t, window, shift)
    w = basa.window_attn_bwd(q, k, v, out, g, lse, window, shift)
    torch.cuda.synchronize()
    for a, b in zip(j[:3], w):
        assert torch.equal(a, b)
    assert all(t.numel() == 0 for t in j[3:])


def test_joint_backward_cuda_core_path(basa):
    """BASA_FLAG_BWD_CUDA_CORES keeps the fp32 CUDA-core kernels reachable for
    bf16; they match the oracle too, and every gradient element there is summed
    by one thread in a fixed order, so two calls give the same bits."""
    shape, window, shift, L = (1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8), 77
    fl = basa.BASA_FLAG_BWD_CUDA_CORES
    a, refs = run_case(basa, shape, 0, window, shift, L, "bf16", seed=191, flags=fl)
    b, _ = run_case(basa, shape, 0, window, shift, L, "bf16", seed=191, flags=fl)
    for x, y, r in zip(a, b, refs):
        assert torch.equal(x, y)
        assert_close(x, r, "bf16", "cuda cores")


def test_joint_backward_tensor_core_repeatability(basa):
    """Tensor cores: dq, dk, dv and dqt are accumulated in a fixed order (same
    bits on every call); the text keys' dkt, dvt are fp32 sums over query-tile
    splits (atomics), so two calls agree to fp32 rounding of the order."""
    shape, window, shift, L = (1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8), 300
    a, _ = run_case(basa, shape, 0, window, shift, L, "bf16", seed=193)
    b, _ = run_case(basa, shape, 0, window, shift, L, "bf16", seed=193)
    for i, (x, y) in enumerate(zip(a, b)):
        if i < 4:
            assert torch.equal(x, y)
        else:
            assert float((x.float() - y.float()).abs().max()) <= 2e-2
