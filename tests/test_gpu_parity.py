"""GPU parity: the CUDA library (through its C ABI) against the CPU fp64 oracle
on the same seeded inputs.  fp32: max-abs <= 1e-5.  bf16: max-abs <= 2e-2 and
relative RMS <= 5e-3."""
import math

import numpy as np
import pytest
import torch

import oracle
from basa_synth import WORKLOADS, make_qkv, workload_inputs
from gpu_util import (assert_close, errors, gather_rows, oracle_params, sample_queries)

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


def _inputs(shape, dtype, seed, q_mult=1.0):
    q, k, v = make_qkv(shape, dtype, seed, seed + 1, seed + 2, q_mult=q_mult)
    return q, k, v


def _run_window(basa, q, k, v, window, shift, pool=(0, 0, 0), lse=True, flags=0):
    dq, dk, dv = (x.cuda() for x in (q, k, v))
    out = basa.window_attn(dq, dk, dv, window, shift, pool, return_lse=lse, flags=flags)
    if lse:
        o, l = out
        torch.cuda.synchronize()
        return o, l
    torch.cuda.synchronize()
    return out, None


def _check_window(basa, shape, dtype, window, shift, pool=(0, 0, 0), seed=1, q_mult=1.0,
                  what="", flags=0):
    q, k, v = _inputs(shape, dtype, seed, q_mult)
    out, lse = _run_window(basa, q, k, v, window, shift, pool, flags=flags)
    prm = oracle_params(shape, window, shift, pool)
    ref, ref_lse = oracle.window_attn(oracle.as_f64(q), oracle.as_f64(k), oracle.as_f64(v),
                                      prm, want_lse=True)
    res = assert_close(out, ref, dtype, what or f"{shape} w{window} s{shift} p{pool}")
    tol = 1e-5 if dtype == "f32" else 2e-2
    lerr = float(np.abs(lse.double().cpu().numpy() - ref_lse).max())
    assert lerr <= tol, f"lse max-abs {lerr}"
    assert basa.get_status() == 0
    return res


# ---------------------------------------------------------------- fp32 (CUDA cores)

def test_fp32_grid16_workload(basa):
    w = WORKLOADS["grid16_f32"]
    q, k, v = workload_inputs(w, 0)
    out, lse = _run_window(basa, q, k, v, w.window, w.shifts[0])
    prm = oracle_params(w.shape(), w.window, w.shifts[0])
    ref, ref_lse = oracle.window_attn(oracle.as_f64(q), oracle.as_f64(k), oracle.as_f64(v),
                                      prm, want_lse=True)
    assert_close(out, ref, "f32", "grid16")
    assert float(np.abs(lse.double().cpu().numpy() - ref_lse).max()) <= 1e-5


@pytest.mark.parametrize("shape,window,shift,pool", [
    ((1, 1, 16, 16, 2, 64), (1, 8, 8), (0, 0, 0), (0, 0, 0)),
    ((1, 1, 16, 16, 2, 64), (1, 8, 8), (0, -3, 5), (1, 4, 4)),
    ((2, 4, 6, 8, 3, 32), (2, 3, 4), (1, 2, 3), (2, 3, 2)),
    ((1, 2, 12, 10, 2, 128), (2, 6, 5), (1, 4, 2), (1, 2, 5)),
    ((1, 1, 8, 12, 1, 64), (1, 8, 12), (0, 3, 7), (0, 0, 0)),
])
def test_fp32_window_variants(basa, shape, window, shift, pool):
    _check_window(basa, shape, "f32", window, shift, pool, seed=7)


@pytest.mark.parametrize("shape", [(1, 1, 16, 16, 2, 64), (2, 3, 5, 7, 2, 32), (1, 1, 9, 11, 1, 128)])
def test_fp32_full_attention(basa, shape):
    q, k, v = _inputs(shape, "f32", 21)
    out, lse = basa.full_attn(q.cuda(), k.cuda(), v.cuda(), return_lse=True)
    B, T, Hg, Wg, H, d = shape
    ref, ref_lse = oracle.full_attn(oracle.as_f64(q), oracle.as_f64(k), oracle.as_f64(v),
                                    oracle_params(shape, (T, Hg, Wg)), want_lse=True)
    assert_close(out, ref, "f32", "full fp32")
    assert float(np.abs(lse.double().cpu().numpy() - ref_lse).max()) <= 1e-5


# ---------------------------------------------------------------- pooling kernel

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pool_kernel(basa, dtype):
    shape = (2, 2, 16, 24, 3, 64 if dtype == "bf16" else 32)
    pool = (2, 4, 3)
    q, k, v = _inputs(shape, dtype, 31)
    kp, vp = basa.pool_kv(k.cuda(), v.cuda(), pool)
    torch.cuda.synchronize()
    prm = oracle_params(shape, (1, 1, 1), pool=pool)
    rk = oracle.pool_kv(oracle.as_f64(k), prm)
    rv = oracle.pool_kv(oracle.as_f64(v), prm)
    gk = kp.double().cpu().numpy()
    gv = vp.double().cpu().numpy()
    if dtype == "f32":
        assert np.abs(gk - rk).max() <= 1e-6 and np.abs(gv - rv).max() <= 1e-6
    else:
        # one rounding to bf16 (relative 2^-8) of an fp32 mean
        assert (np.abs(gk - rk) <= np.abs(rk) * 2.0 ** -8 + 1e-6).all()
        assert (np.abs(gv - rv) <= np.abs(rv) * 2.0 ** -8 + 1e-6).all()


# ---------------------------------------------------------------- bf16 (tcgen05)

BF16_CASES = [
    # 2D, 16 x 16 windows, the shifts of the image workloads
    ((1, 1, 64, 64, 2, 128), (1, 16, 16), (0, 0, 0), (0, 0, 0)),
    ((1, 1, 64, 64, 2, 128), (1, 16, 16), (0, 8, 8), (0, 0, 0)),
    ((1, 1, 64, 64, 2, 128), (1, 16, 16), (0, 8, 0), (0, 0, 0)),
    ((2, 1, 32, 48, 2, 128), (1, 16, 16), (0, -8, 24), (0, 0, 0)),
    # head dim 64
    ((1, 1, 32, 32, 3, 64), (1, 16, 16), (0, 8, 8), (0, 0, 0)),
    # a window of one 128-row tile (odd tile count per window) and of 64 tokens
    ((1, 1, 32, 32, 2, 128), (1, 8, 16), (0, 4, 8), (0, 0, 0)),
    ((1, 1, 16, 16, 2, 128), (1, 8, 8), (0, 4, 0), (0, 0, 0)),
    # 3D video windows: 7 x 9 x 16 with a 112-row tile, wrapped on every axis
    ((1, 14, 18, 32, 2, 128), (7, 9, 16), (3, 4, 8), (0, 0, 0)),
    ((1, 14, 18, 32, 1, 64), (7, 9, 16), (0, 0, 0), (0, 0, 0)),
    # pooled global memory: 64 pooled tokens (ragged tile) and 256 (two tiles)
    ((1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8), (1, 4, 4)),
    ((2, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 0), (1, 2, 2)),
    ((1, 14, 18, 32, 1, 128), (7, 9, 16), (3, 4, 8), (7, 3, 4)),
]


@pytest.mark.parametrize("shape,window,shift,pool", BF16_CASES)
def test_bf16_window(basa, shape, window, shift, pool):
    _check_window(basa, shape, "bf16", window, shift, pool, seed=11)


def test_bf16_large_logits(basa):
    # logits scaled x8 per head: the running max moves across key tiles
    _check_window(basa, (1, 1, 32, 32, 2, 128), "bf16", (1, 16, 16), (0, 8, 8), (1, 4, 4),
                  seed=13, q_mult=8.0)


@pytest.mark.parametrize("shape", [(1, 1, 16, 20, 2, 128), (2, 1, 8, 16, 2, 64),
                                   (1, 1, 32, 32, 2, 128)])
def test_bf16_full_attention(basa, shape):
    q, k, v = _inputs(shape, "bf16", 41)
    out, lse = basa.full_attn(q.cuda(), k.cuda(), v.cuda(), return_lse=True)
    torch.cuda.synchronize()
    B, T, Hg, Wg, H, d = shape
    ref, ref_lse = oracle.full_attn(oracle.as_f64(q), oracle.as_f64(k), oracle.as_f64(v),
                                    oracle_params(shape, (T, Hg, Wg)), want_lse=True)
    assert_close(out, ref, "bf16", "full bf16")
    assert float(np.abs(lse.double().cpu().numpy() - ref_lse).max()) <= 2e-2
    assert basa.get_status() == 0


def test_bf16_window_gm_matches_window_attn(basa):
    shape, window, shift, pool = (1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8), (1, 4, 4)
    q, k, v = (x.cuda() for x in _inputs(shape, "bf16", 51))
    kp, vp = basa.pool_kv(k, v, pool)
    a = basa.window_attn(q, k, v, window, shift, pool)
    b = basa.window_attn_gm(q, k, v, kp, vp, window, shift, pool)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_bf16_deterministic_and_roll_commutes(basa):
    shape, window, shift = (1, 1, 64, 64, 2, 128), (1, 16, 16), (0, 8, 8)
    q, k, v = (x.cuda() for x in _inputs(shape, "bf16", 61))
    a = basa.window_attn(q, k, v, window, shift)
    b = basa.window_attn(q, k, v, window, shift)
    torch.cuda.synchronize()
    assert torch.equal(a, b), "repeated runs differ"
    dims = (2, 3)
    r = basa.window_attn(*(torch.roll(x, (-8, -8), dims) for x in (q, k, v)), window, (0, 0, 0))
    back = torch.roll(r, (8, 8), dims)
    maxabs, relrms = errors(back, a.double().cpu().numpy())
    assert maxabs <= 2e-2 and relrms <= 5e-3


# ---------------------------------------------------------------- the full-size workloads

def _workload_sampled(basa, name, block, nsample=384):
    w = WORKLOADS[name]
    q, k, v = workload_inputs(w, block)
    shift = w.shifts[block]
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    out, lse = basa.window_attn(dq, dk, dv, w.window, shift, w.pool, return_lse=True)
    torch.cuda.synchronize()
    assert basa.get_status() == 0
    sel = sample_queries(w.shape(), nsample, 1000 + block)
    prm = oracle_params(w.shape(), w.window, shift, w.pool)
    ref, ref_lse = oracle.window_attn(oracle.as_f64(q), oracle.as_f64(k), oracle.as_f64(v), prm,
                                      want_lse=True, select=sel)
    got = gather_rows(out, sel)
    assert_close(got, ref, w.dtype, f"{name} block {block}")
    B, T, Hg, Wg, H, d = w.shape()
    got_lse = lse[torch.as_tensor(sel[:, 0]), torch.as_tensor(sel[:, 2]), torch.as_tensor(sel[:, 1])]
    assert float(np.abs(got_lse.double().cpu().numpy() - ref_lse).max()) <= 2e-2
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("block", [0, 1])
def test_flux1024_sampled(basa, block):
    _workload_sampled(basa, "flux1024", block)


def test_flux2048_sampled(basa):
    _workload_sampled(basa, "flux2048", 0)


def test_wan_video_sampled(basa):
    _workload_sampled(basa, "wan_video", 0, nsample=192)


@pytest.mark.parametrize("block", [0, 1, 2, 3])
def test_flux2048_gm4_sampled(basa, block):
    _workload_sampled(basa, "flux2048_gm4", block, nsample=192)


# ---------------------------------------------------------------- every element at full size

def _workload_rows(basa, name, block, heads=None, batches=None):
    """Every output row and lse of the listed heads and batches of a full-size
    workload (default: all of them) against the oracle, in the launch
    configuration the benchmark times."""
    w = WORKLOADS[name]
    q, k, v = workload_inputs(w, block)
    shift = w.shifts[block]
    B, T, Hg, Wg, H, d = w.shape()
    N = w.N
    heads = list(range(H)) if heads is None else list(heads)
    batches = list(range(B)) if batches is None else list(batches)
    out, lse = basa.window_attn(q.cuda(), k.cuda(), v.cuda(), w.window, shift, w.pool,
                                return_lse=True)
    torch.cuda.synchronize()
    assert basa.get_status() == 0
    prm = oracle_params(w.shape(), w.window, shift, w.pool)
    qf, kf, vf = oracle.as_f64(q), oracle.as_f64(k), oracle.as_f64(v)
    kp = vp = None
    if w.P:
        kp, vp = oracle.pool_kv(kf, prm), oracle.pool_kv(vf, prm)
    hsel = np.asarray(heads, dtype=np.int64)
    for b in batches:
        # rows (b, n, h), n outer and h inner: the order of out[b, n, heads]
        sel = np.stack([np.full(N * len(heads), b, dtype=np.int64),
                        np.repeat(np.arange(N, dtype=np.int64), len(heads)),
                        np.tile(hsel, N)], axis=1)
        ref, ref_lse = oracle.window_attn(qf, kf, vf, prm, kp=kp, vp=vp, want_lse=True,
                                          select=sel)
        got = out.reshape(B, N, H, d)[b][:, torch.as_tensor(hsel, device=out.device)]
        assert_close(got.reshape(-1, d), ref, w.dtype, f"{name} block {block} batch {b}")
        got_lse = lse[b][torch.as_tensor(hsel, device=lse.device)].t().reshape(-1)
        lerr = float(np.abs(got_lse.double().cpu().numpy() - ref_lse).max())
        assert lerr <= 2e-2, f"{name} block {block} batch {b}: lse max-abs {lerr}"
    assert torch.isfinite(out).all()


def test_flux2048_every_element(basa):
    """The benchmark's workload: all 24 heads, all 16384 queries, and the lse."""
    _workload_rows(basa, "flux2048", 0)


def test_flux2048_gm4_block_every_element(basa):
    """One whole block of the four-block schedule with 1024 pooled tokens (both
    batches, every head and query); the last block's shift, as benchmarked."""
    _workload_rows(basa, "flux2048_gm4", 3)


def test_wan_video_two_heads_every_element(basa):
    """Every query of two of Wan's 40 heads (the first and the last)."""
    _workload_rows(basa, "wan_video", 0, heads=[0, 39])
