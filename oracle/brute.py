"""Dense-mask brute force for tiny grids (test infrastructure only).

A second, independent restatement of shifted local window attention: build the
N x N "same window" mask from the window-id reading (token x on an axis of size G
with window w and shift s lies in window floor(((x - s) mod G) / w)), append the
pooled keys as columns that every query sees, and take one masked softmax per
query row in float64.  Pooling here is a numpy reshape-mean, written apart from
the C oracle's loop.

Sources: "BASA: Backend-Agnostic Sparse Attention for Fast High-Resolution
Diffusion Transformers" (zhichai.net topic 178635722), "The BASA Method"; the
forum review of the same paper (reply 178634520), four-part method list
(K/V-pooled global memory).
"""
from __future__ import annotations

import math

import numpy as np


def window_ids(G: int, w: int, s: int, pad: bool = False) -> np.ndarray:
    """Window index of every coordinate 0..G-1 on one axis.  With ``pad`` the
    axis is first padded to the next multiple of w (padding holds no token) and
    the shift rolls the padded axis."""
    x = np.arange(G)
    Gp = -(-G // w) * w if pad else G
    return ((x - s) % Gp) // w


def _pool(x: np.ndarray, pool) -> np.ndarray:
    B, T, Hg, Wg, H, d = x.shape
    pt, ph, pw = pool
    r = x.reshape(B, T // pt, pt, Hg // ph, ph, Wg // pw, pw, H, d)
    return r.mean(axis=(2, 4, 6))


def brute_window_attn(q, k, v, window, shift=(0, 0, 0), pool=(0, 0, 0), scale=None,
                      want_lse=False, pad=False):
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, T, Hg, Wg, H, d = q.shape
    N = T * Hg * Wg
    sc = 1.0 / math.sqrt(d) if scale is None else scale
    it = window_ids(T, window[0], shift[0], pad)
    iy = window_ids(Hg, window[1], shift[1], pad)
    ix = window_ids(Wg, window[2], shift[2], pad)
    wid = np.stack(np.meshgrid(it, iy, ix, indexing="ij"), axis=-1).reshape(N, 3)
    mask = np.all(wid[:, None, :] == wid[None, :, :], axis=-1)  # [N, N]
    qf = q.reshape(B, N, H, d).transpose(0, 2, 1, 3)
    kf = k.reshape(B, N, H, d).transpose(0, 2, 1, 3)
    vf = v.reshape(B, N, H, d).transpose(0, 2, 1, 3)
    if tuple(pool) != (0, 0, 0):
        kp = _pool(k, pool)
        vp = _pool(v, pool)
        P = kp.shape[1] * kp.shape[2] * kp.shape[3]
        kf = np.concatenate([kf, kp.reshape(B, P, H, d).transpose(0, 2, 1, 3)], axis=2)
        vf = np.concatenate([vf, vp.reshape(B, P, H, d).transpose(0, 2, 1, 3)], axis=2)
        mask = np.concatenate([mask, np.ones((N, P), dtype=bool)], axis=1)
    z = sc * np.einsum("bhnc,bhjc->bhnj", qf, kf)
    z = np.where(mask[None, None], z, -np.inf)
    mx = z.max(axis=-1, keepdims=True)
    e = np.exp(z - mx)
    den = e.sum(axis=-1, keepdims=True)
    o = np.einsum("bhnj,bhjc->bhnc", e / den, vf)
    out = o.transpose(0, 2, 1, 3).reshape(B, T, Hg, Wg, H, d)
    if want_lse:
        lse = (mx + np.log(den))[..., 0]  # [B, H, N]
        return out, lse
    return out


def brute_joint_attn(q, k, v, qt, kt, vt, window, shift=(0, 0, 0), scale=None, want_lse=False,
                     pad=False):
    """Joint text + image attention as one dense masked softmax over the
    concatenated sequence [N image tokens, L text tokens]: image-image pairs keep
    the same-window mask, every pair that involves a text token is allowed."""
    q, k, v, qt, kt, vt = (np.asarray(x, dtype=np.float64) for x in (q, k, v, qt, kt, vt))
    B, T, Hg, Wg, H, d = q.shape
    N, L = T * Hg * Wg, qt.shape[1]
    sc = 1.0 / math.sqrt(d) if scale is None else scale
    it = window_ids(T, window[0], shift[0], pad)
    iy = window_ids(Hg, window[1], shift[1], pad)
    ix = window_ids(Wg, window[2], shift[2], pad)
    wid = np.stack(np.meshgrid(it, iy, ix, indexing="ij"), axis=-1).reshape(N, 3)
    mask = np.ones((N + L, N + L), dtype=bool)
    mask[:N, :N] = np.all(wid[:, None, :] == wid[None, :, :], axis=-1)
    qa = np.concatenate([q.reshape(B, N, H, d), qt], axis=1).transpose(0, 2, 1, 3)
    ka = np.concatenate([k.reshape(B, N, H, d), kt], axis=1).transpose(0, 2, 1, 3)
    va = np.concatenate([v.reshape(B, N, H, d), vt], axis=1).transpose(0, 2, 1, 3)
    z = sc * np.einsum("bhnc,bhjc->bhnj", qa, ka)
    z = np.where(mask[None, None], z, -np.inf)
    mx = z.max(axis=-1, keepdims=True)
    e = np.exp(z - mx)
    den = e.sum(axis=-1, keepdims=True)
    o = np.einsum("bhnj,bhjc->bhnc", e / den, va).transpose(0, 2, 1, 3)  # [B, N+L, H, d]
    out = o[:, :N].reshape(B, T, Hg, Wg, H, d)
    out_t = o[:, N:]
    if want_lse:
        lse = (mx + np.log(den))[..., 0]  # [B, H, N+L]
        return out, out_t, lse[:, :, :N], lse[:, :, N:]
    return out, out_t
