"""Helpers shared by the GPU parity tests: tolerance checks and oracle calls."""
import math

import numpy as np
import torch

import oracle

# Tolerances: fp32 max-abs 1e-5; bf16 max-abs 2e-2 and relative RMS 5e-3.
TOL_F32 = 1e-5
TOL_BF16_MAXABS = 2e-2
TOL_BF16_RELRMS = 5e-3


def errors(gpu, ref):
    g = gpu.detach().to("cpu", torch.float64).numpy() if isinstance(gpu, torch.Tensor) else gpu
    ref = np.asarray(ref, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64).reshape(ref.shape)
    assert np.isfinite(g).all(), "non-finite GPU output"
    err = np.abs(g - ref)
    maxabs = float(err.max()) if err.size else 0.0
    denom = float(np.sqrt((ref ** 2).sum()))
    relrms = float(np.sqrt((err ** 2).sum()) / denom) if denom > 0 else 0.0
    return maxabs, relrms


def assert_close(gpu, ref, dtype, what=""):
    maxabs, relrms = errors(gpu, ref)
    if dtype in ("f32", torch.float32):
        assert maxabs <= TOL_F32, f"{what}: fp32 max-abs {maxabs:.3e} > {TOL_F32}"
    else:
        assert maxabs <= TOL_BF16_MAXABS, f"{what}: bf16 max-abs {maxabs:.3e}"
        assert relrms <= TOL_BF16_RELRMS, f"{what}: bf16 rel-RMS {relrms:.3e}"
    return maxabs, relrms


def oracle_params(shape, window, shift=(0, 0, 0), pool=(0, 0, 0), scale=None):
    B, T, Hg, Wg, H, d = shape
    return oracle.OracleParams(B, T, Hg, Wg, H, d, tuple(window), tuple(shift), tuple(pool), scale)


def sample_queries(shape, n, seed):
    B, T, Hg, Wg, H, d = shape
    N = T * Hg * Wg
    g = np.random.Generator(np.random.PCG64(seed))
    b = g.integers(0, B, n)
    t = g.integers(0, N, n)
    h = g.integers(0, H, n)
    # always include the grid corners (wrapped windows) and the last token
    extra = np.array([[0, 0, 0], [B - 1, N - 1, H - 1], [0, N - 1, 0], [B - 1, 0, H - 1]])
    return np.concatenate([np.stack([b, t, h], axis=1), extra]).astype(np.int64)


def gather_rows(out, sel):
    """Rows out[b, n, h, :] of a [B, T, Hg, Wg, H, d] tensor for (b, n, h) triples."""
    B, T, Hg, Wg, H, d = out.shape
    flat = out.reshape(B, T * Hg * Wg, H, d)
    idx_b = torch.as_tensor(sel[:, 0], device=out.device)
    idx_n = torch.as_tensor(sel[:, 1], device=out.device)
    idx_h = torch.as_tensor(sel[:, 2], device=out.device)
    return flat[idx_b, idx_n, idx_h]
