"""Invariants of the GPU outputs that hold at any size, from the method's
definition ("BASA: Backend-Agnostic Sparse Attention for Fast High-Resolution
Diffusion Transformers", zhichai.net topic 178635722, "The BASA Method": each
token attends within its own cyclically shifted window, and the shift lets
tokens on either side of a window border meet in a later block):

- support: changing one token's value changes exactly the outputs of the
  queries of its window, on its head, and nothing else (bit for bit);
- two blocks, (0, 0) then (w/2, w/2): the change reaches the union of the
  shifted windows of the first window's tokens, across the border;
- linearity in v, constant v, and q = 0 (uniform weights over window and
  pooled keys, the forum review's K/V-pooled global memory) closed forms.

Window membership here is written out from the reading used throughout:
token x on an axis of size G with window w and shift s is in window
floor(((x - s) mod G) / w)."""
import numpy as np
import pytest
import torch

from basa_synth import make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def basa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_diffusion_basa_b200 import build
    build.build()
    import sparse_attention_diffusion_basa_b200 as m
    return m


def window_of(T, Hg, Wg, window, shift):
    """[N, 3] window index of every token of the grid."""
    t, y, x = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(Wg), indexing="ij")
    ids = [((c - s) % G) // w for c, s, G, w in zip((t, y, x), shift, (T, Hg, Wg), window)]
    return np.stack([i.reshape(-1) for i in ids], axis=1)


def same_window(wid, n):
    return np.all(wid == wid[n], axis=1)


def changed_tokens(a, b, head):
    """Tokens whose output row on `head` differs between a and b, [B, T, Hg, Wg, H, d]."""
    B, T, Hg, Wg, H, d = a.shape
    diff = (a != b).reshape(B, T * Hg * Wg, H, d).any(dim=-1)[0]  # [N, H]
    return diff[:, head].cpu().numpy(), diff


CASES = [  # shape, window, shift, dtype
    ((1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8), "bf16"),
    ((1, 6, 10, 16, 2, 64), (3, 5, 8), (1, 2, 0), "bf16"),
    ((1, 1, 16, 16, 2, 64), (1, 8, 8), (0, 4, 4), "f32"),
]


@pytest.mark.parametrize("shape,window,shift,dtype", CASES)
def test_support_is_the_shifted_window(basa, shape, window, shift, dtype):
    B, T, Hg, Wg, H, d = shape
    q, k, v = (x.cuda() for x in make_qkv(shape, dtype, 201, 202, 203))
    base = basa.window_attn(q, k, v, window, shift)
    wid = window_of(T, Hg, Wg, window, shift)
    N = T * Hg * Wg
    for n in (0, N - 1, N // 2 + 3):  # grid corners (wrapped windows) and an inner token
        v2 = v.clone()
        v2.view(B, N, H, d)[0, n, 1] += 1000.0
        out = basa.window_attn(q, k, v2, window, shift)
        torch.cuda.synchronize()
        got, diff = changed_tokens(base, out, 1)
        assert np.array_equal(got, same_window(wid, n)), f"token {n}"
        assert not diff[:, 0].any(), "another head changed"


def test_two_blocks_reach_across_the_window_border(basa):
    """fp32: block 1 unshifted, block 2 shifted by half a window, block 2's values
    are block 1's outputs; a change of one value reaches exactly the tokens that
    share a shifted window with some token of its unshifted window."""
    shape, window = (1, 1, 32, 32, 2, 64), (1, 8, 8)
    s0, s1 = (0, 0, 0), (0, 4, 4)
    B, T, Hg, Wg, H, d = shape
    q, k, v = (x.cuda() for x in make_qkv(shape, "f32", 211, 212, 213))
    two = lambda vv: basa.window_attn(q, k, basa.window_attn(q, k, vv, window, s0), window, s1)
    base = two(v)
    N = T * Hg * Wg
    w0, w1 = window_of(T, Hg, Wg, window, s0), window_of(T, Hg, Wg, window, s1)
    for n in (0, 9 * Wg + 9, N - 1):
        v2 = v.clone()
        v2.view(B, N, H, d)[0, n, 0] += 10.0
        out = two(v2)
        torch.cuda.synchronize()
        got, _ = changed_tokens(base, out, 0)
        first = same_window(w0, n)
        expect = np.zeros(N, dtype=bool)
        for u in np.nonzero(first)[0]:
            expect |= same_window(w1, u)
        assert np.array_equal(got, expect), f"token {n}"
        assert (expect & ~first).any()  # the reach crosses the border of the first window


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_linear_in_v(basa, dtype):
    shape, window, shift = (1, 1, 32, 32, 2, 128 if dtype == "bf16" else 64), (1, 16, 16), (0, 8, 8)
    q, k, v1 = (x.cuda() for x in make_qkv(shape, dtype, 221, 222, 223))
    _, _, v2 = (x.cuda() for x in make_qkv(shape, dtype, 224, 225, 226))
    a = basa.window_attn(q, k, v1, window, shift).double()
    b = basa.window_attn(q, k, v2, window, shift).double()
    c = basa.window_attn(q, k, (v1.double() + v2.double()).to(v1.dtype), window, shift).double()
    torch.cuda.synchronize()
    tol = 1e-5 if dtype == "f32" else 4e-2  # the sum of two bf16-rounded outputs
    assert float((a + b - c).abs().max()) <= tol


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_constant_values_come_back(basa, dtype):
    """Softmax weights sum to one: v = c per head gives out = c (bf16: within
    the rounding of P and of the output, 2^-7 relative to |c| <= 1.5)."""
    shape, window, shift = (1, 1, 32, 32, 2, 128 if dtype == "bf16" else 64), (1, 16, 16), (0, 8, 8)
    q, k, _ = (x.cuda() for x in make_qkv(shape, dtype, 231, 232, 233))
    c = torch.tensor([1.5, -0.75], device="cuda").view(1, 1, 1, 1, 2, 1)
    v = (torch.ones(shape, device="cuda") * c).to(q.dtype)
    out = basa.window_attn(q, k, v, window, shift).double()
    torch.cuda.synchronize()
    # fp32: the suite's 1e-5 bound (summing 256 weights in fp32 costs about 1e-6)
    tol = 1e-5 if dtype == "f32" else 2.0 ** -7 * 1.5
    assert float((out - c.double()).abs().max()) <= tol


def test_zero_queries_average_window_and_pooled_values(basa):
    """q = 0: every key gets the same weight, so out is the mean of the m window
    values and the P pooled values (means of their cells), computed here with
    plain tensor means; fp32."""
    shape, window, shift, pool = (1, 1, 16, 16, 2, 64), (1, 8, 8), (0, 4, 4), (1, 4, 4)
    B, T, Hg, Wg, H, d = shape
    _, k, v = (x.cuda() for x in make_qkv(shape, "f32", 241, 242, 243))
    q = torch.zeros(shape, device="cuda")
    out = basa.window_attn(q, k, v, window, shift, pool)
    torch.cuda.synchronize()
    vc = v.double().cpu()
    cells = vc.reshape(B, T, Hg // 4, 4, Wg // 4, 4, H, d).mean(dim=(3, 5)).reshape(B, -1, H, d)
    wid = window_of(T, Hg, Wg, window, shift)
    vf = vc.reshape(B, T * Hg * Wg, H, d)
    m, P = 64, cells.shape[1]
    for n in (0, 37, 255):
        member = torch.as_tensor(same_window(wid, n))
        ref = (vf[0, member].sum(0) + cells[0].sum(0)) / (m + P)
        got = out.reshape(B, -1, H, d)[0, n].double().cpu()
        assert float((got - ref).abs().max()) <= 1e-5
