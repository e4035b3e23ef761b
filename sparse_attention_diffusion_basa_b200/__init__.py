"""Shifted local window attention for Diffusion Transformer tokens on B200.

A thin Python binding over the C ABI of ``include/basa.h``: it checks tensor
placement, allocates outputs with torch (device memory only) and passes raw
pointers and the current CUDA stream to the library.  Every step of the
computation runs in the library's CUDA kernels; there is no CPU or PyTorch
fallback, and calls fail loudly when the library is missing.

Tensors use the layout ``[B, T, Hg, Wg, H, d]``; ``window``, ``shift`` and
``pool`` are (t, rows, columns) triples.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence, Tuple

import torch

from . import _lib
from ._lib import BasaError, BasaParams, BASA_F32, BASA_BF16, BASA_FP8_E4M3  # noqa: F401
from ._lib import BASA_FLAG_PAD_GRID, BASA_FLAG_BWD_CUDA_CORES  # noqa: F401

__all__ = ["window_attn", "window_attn_gm", "full_attn", "joint_attn", "window_attn_bwd",
           "joint_attn_bwd",
           "pool_kv", "workspace_size", "bwd_workspace_size", "joint_workspace_size",
           "joint_bwd_workspace_size", "get_status", "window_tiles", "make_params", "BasaError",
           "library_path", "BASA_FLAG_PAD_GRID", "BASA_FLAG_BWD_CUDA_CORES"]

library_path = _lib.LIB_PATH

_DT = {torch.float32: BASA_F32, torch.bfloat16: BASA_BF16, torch.float8_e4m3fn: BASA_FP8_E4M3}


def _triple(x, name) -> Tuple[int, int, int]:
    t = tuple(int(v) for v in x)
    if len(t) != 3:
        raise ValueError(f"{name} must have 3 entries (t, rows, columns), got {x!r}")
    return t


def make_params(shape: Sequence[int], dtype, window=(1, 1, 1), shift=(0, 0, 0),
                pool=(0, 0, 0), scale: Optional[float] = None, flags: int = 0,
                wait_timeout_ms: int = 0, hkv: int = 0, descale=(0.0, 0.0, 0.0)) -> BasaParams:
    B, T, Hg, Wg, H, d = (int(s) for s in shape)
    if isinstance(dtype, torch.dtype):
        dtype = _DT[dtype]
    w, s, p = _triple(window, "window"), _triple(shift, "shift"), _triple(pool, "pool")
    dq, dk, dv = (float(x) for x in descale)
    return BasaParams(B, H, T, Hg, Wg, d, *w, *s, *p, float(scale or 0.0), int(dtype),
                      int(flags), int(wait_timeout_ms), int(hkv), dq, dk, dv)


def _out_like(q):
    """Output tensor of an attention call: bf16 for e4m3 inputs, else q's dtype."""
    if q.dtype == torch.float8_e4m3fn:
        return torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    return torch.empty_like(q)


def _kv_heads(q, k, v) -> int:
    """K/V head count for grouped-query attention (0 when it equals q's)."""
    if k.shape != v.shape:
        raise ValueError("k and v must have the same shape")
    if k.shape[:-2] != q.shape[:-2] or k.shape[-1] != q.shape[-1]:
        raise ValueError(f"k {tuple(k.shape)} must match q {tuple(q.shape)} except in heads")
    H, Hkv = q.shape[-2], k.shape[-2]
    if Hkv == 0 or H % Hkv:
        raise ValueError(f"q heads {H} must be a multiple of k/v heads {Hkv}")
    return 0 if Hkv == H else Hkv


def _check_inputs(*ts):
    ref = ts[0]
    for t in ts:
        if not isinstance(t, torch.Tensor):
            raise TypeError("expected torch tensors")
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device")
        if t.dtype not in _DT:
            raise TypeError(f"unsupported dtype {t.dtype}")
        if t.dtype != ref.dtype or t.device != ref.device:
            raise ValueError("q, k, v must share dtype and device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, T, Hg, Wg, H, d]")
        if t.dim() != 6:
            raise ValueError("tensors must have 6 dims [B, T, Hg, Wg, H, d]")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor, stream=None):
    s = stream if stream is not None else torch.cuda.current_stream(t.device)
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(shape, dtype, window, shift=(0, 0, 0), pool=(0, 0, 0), hkv=0) -> int:
    return int(_lib.load().basa_workspace_size(
        ctypes.byref(make_params(shape, dtype, window, shift, pool, hkv=hkv))))


def bwd_workspace_size(shape, dtype, window, shift=(0, 0, 0), pool=(0, 0, 0), hkv=0) -> int:
    """Bytes of device workspace that window_attn_bwd needs for this problem."""
    return int(_lib.load().basa_bwd_workspace_size(
        ctypes.byref(make_params(shape, dtype, window, shift, pool, hkv=hkv))))


def joint_workspace_size(shape, dtype, window, shift, L, hkv=0) -> int:
    """Bytes of device workspace joint_attn uses to split its text-query pass (0: none)."""
    return int(_lib.load().basa_joint_workspace_size(
        ctypes.byref(make_params(shape, dtype, window, shift, (0, 0, 0), hkv=hkv)), int(L)))


def joint_bwd_workspace_size(shape, dtype, window, shift, L, hkv=0, flags=0) -> int:
    """Bytes of device workspace joint_attn_bwd needs (D of the image and text rows)."""
    return int(_lib.load().basa_joint_bwd_workspace_size(
        ctypes.byref(make_params(shape, dtype, window, shift, (0, 0, 0), flags=flags, hkv=hkv)),
        int(L)))


def pool_kv(k: torch.Tensor, v: torch.Tensor, pool, out=None, stream=None):
    """Mean-pool K and V over pt x ph x pw cells -> (kp, vp) [B, T/pt, Hg/ph, Wg/pw, H, d].

    ``out`` may give the (kp, vp) tensors to write into."""
    _check_inputs(k, v)
    B, T, Hg, Wg, H, d = k.shape
    pt, ph, pw = _triple(pool, "pool")
    if min(pt, ph, pw) <= 0 or T % pt or Hg % ph or Wg % pw:
        raise ValueError(f"pool {pool} must be positive and divide the grid {(T, Hg, Wg)}")
    shape = (B, T // pt, Hg // ph, Wg // pw, H, d)
    if out is None:
        kp = torch.empty(shape, dtype=k.dtype, device=k.device)
        vp = torch.empty_like(kp)
    else:
        kp, vp = out
        _check_inputs(k, kp, vp)
        if tuple(kp.shape) != shape or tuple(vp.shape) != shape:
            raise ValueError(f"pooled outputs must have shape {shape}")
    prm = make_params(k.shape, k.dtype, (1, 1, 1), (0, 0, 0), (pt, ph, pw))
    lib = _lib.load()
    with torch.cuda.device(k.device):
        _lib.check(lib.basa_pool_kv(_ptr(k), _ptr(v), _ptr(kp), _ptr(vp), ctypes.byref(prm),
                                    _stream(k, stream)), "basa_pool_kv")
    return kp, vp


def window_attn(q, k, v, window, shift=(0, 0, 0), pool=(0, 0, 0), scale=None,
                return_lse=False, out=None, workspace=None, flags=0, wait_timeout_ms=0,
                stream=None, descale=(0.0, 0.0, 0.0)):
    """Shifted local window attention (plus pooled global memory when pool != 0).

    e4m3 inputs (torch.float8_e4m3fn, d = 128, no pool): each tensor's values
    times its factor in ``descale`` (q, k, v; 0 = 1); the output is bf16."""
    _check_inputs(q, k, v)
    hkv = _kv_heads(q, k, v)
    prm = make_params(q.shape, q.dtype, window, shift, pool, scale, flags, wait_timeout_ms, hkv,
                      descale)
    lib = _lib.load()
    out = _out_like(q) if out is None else out
    B, T, Hg, Wg, H, d = q.shape
    lse = torch.empty((B, H, T * Hg * Wg), dtype=torch.float32, device=q.device) if return_lse else None
    need = int(lib.basa_workspace_size(ctypes.byref(prm)))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        _lib.check(lib.basa_window_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                        _ptr(workspace) if need else None, ctypes.byref(prm),
                                        _stream(q, stream)), "basa_window_attn")
    return (out, lse) if return_lse else out


def window_attn_gm(q, k, v, kp, vp, window, shift=(0, 0, 0), pool=(1, 1, 1), scale=None,
                   return_lse=False, out=None, flags=0, stream=None):
    """Window attention with caller-supplied pooled global memory kp, vp."""
    _check_inputs(q, k, v, kp, vp)
    hkv = _kv_heads(q, k, v)
    prm = make_params(q.shape, q.dtype, window, shift, pool, scale, flags, hkv=hkv)
    lib = _lib.load()
    out = torch.empty_like(q) if out is None else out
    B, T, Hg, Wg, H, d = q.shape
    lse = torch.empty((B, H, T * Hg * Wg), dtype=torch.float32, device=q.device) if return_lse else None
    with torch.cuda.device(q.device):
        _lib.check(lib.basa_window_attn_gm(_ptr(q), _ptr(k), _ptr(v), _ptr(kp), _ptr(vp),
                                           _ptr(out), _ptr(lse), ctypes.byref(prm),
                                           _stream(q, stream)), "basa_window_attn_gm")
    return (out, lse) if return_lse else out


def full_attn(q, k, v, scale=None, return_lse=False, out=None, flags=0, stream=None,
              descale=(0.0, 0.0, 0.0)):
    """Full softmax attention over all grid tokens (one window covering the grid);
    e4m3 inputs as in window_attn."""
    _check_inputs(q, k, v)
    hkv = _kv_heads(q, k, v)
    prm = make_params(q.shape, q.dtype, (1, 1, 1), (0, 0, 0), (0, 0, 0), scale, flags, hkv=hkv,
                      descale=descale)
    lib = _lib.load()
    out = _out_like(q) if out is None else out
    B, T, Hg, Wg, H, d = q.shape
    lse = torch.empty((B, H, T * Hg * Wg), dtype=torch.float32, device=q.device) if return_lse else None
    with torch.cuda.device(q.device):
        _lib.check(lib.basa_full_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                      ctypes.byref(prm), _stream(q, stream)), "basa_full_attn")
    return (out, lse) if return_lse else out


def joint_attn(q, k, v, qt, kt, vt, window, shift=(0, 0, 0), scale=None, return_lse=False,
               out=None, out_t=None, workspace=None, flags=0, stream=None):
    """Joint text + image attention with shifted windows for the image queries.

    q, k, v: image tokens [B, T, Hg, Wg, H, d]; qt, kt, vt: text tokens [B, L, H, d].
    Image queries attend to their window plus every text token; text queries
    attend to every token.  Returns (out, out_t) or (out, out_t, lse, lse_t).
    ``workspace`` (uint8 device tensor) is allocated here when the text pass
    splits its key range and none is given."""
    _check_inputs(q, k, v)
    hkv = _kv_heads(q, k, v)
    for t in (qt, kt, vt):
        if not isinstance(t, torch.Tensor) or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("text tensors must be torch tensors with q's dtype and device")
        if not t.is_contiguous():
            raise ValueError("text tensors must be contiguous [B, L, H, d]")
    B, T, Hg, Wg, H, d = q.shape
    if qt.dim() != 4 or qt.shape[0] != B or qt.shape[2:] != (H, d):
        raise ValueError(f"text tokens must be [B, L, H, d] = [{B}, L, {H}, {d}], got {tuple(qt.shape)}")
    if kt.shape != vt.shape or kt.shape != (qt.shape[0], qt.shape[1], k.shape[4], qt.shape[3]):
        raise ValueError("kt and vt must be [B, L, Hkv, d] with qt's B, L, d and k's heads")
    L = qt.shape[1]
    prm = make_params(q.shape, q.dtype, window, shift, (0, 0, 0), scale, flags, hkv=hkv)
    lib = _lib.load()
    out = torch.empty_like(q) if out is None else out
    out_t = torch.empty_like(qt) if out_t is None else out_t
    lse = lse_t = None
    if return_lse:
        lse = torch.empty((B, H, T * Hg * Wg), dtype=torch.float32, device=q.device)
        lse_t = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        need = int(lib.basa_joint_workspace_size(ctypes.byref(prm), int(L)))
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        if need and (workspace.device != q.device or workspace.numel() * workspace.element_size() < need):
            raise ValueError(f"workspace must hold {need} bytes on {q.device}")
        _lib.check(lib.basa_joint_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(qt), _ptr(kt), _ptr(vt),
                                       int(L), _ptr(out), _ptr(out_t), _ptr(lse), _ptr(lse_t),
                                       _ptr(workspace) if need else None, ctypes.byref(prm),
                                       _stream(q, stream)), "basa_joint_attn")
    return (out, out_t, lse, lse_t) if return_lse else (out, out_t)


def window_attn_bwd(q, k, v, out, dout, lse, window, shift=(0, 0, 0), pool=(0, 0, 0),
                    scale=None, workspace=None, flags=0, stream=None):
    """Gradients (dq, dk, dv) of window attention for the output gradient ``dout``.

    ``out`` and ``lse`` are the forward call's output and log-sum-exp; ``pool``
    the forward's pooled cell (its pooled K, V are recomputed in the workspace)."""
    _check_inputs(q, k, v, out, dout)
    hkv = _kv_heads(q, k, v)
    if lse is None or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be the forward's contiguous fp32 log-sum-exp")
    prm = make_params(q.shape, q.dtype, window, shift, pool, scale, flags, hkv=hkv)
    lib = _lib.load()
    need = int(lib.basa_bwd_workspace_size(ctypes.byref(prm)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    with torch.cuda.device(q.device):
        _lib.check(lib.basa_window_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout),
                                            _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                                            _ptr(workspace), ctypes.byref(prm),
                                            _stream(q, stream)), "basa_window_attn_bwd")
    return dq, dk, dv


def joint_attn_bwd(q, k, v, qt, kt, vt, out, out_t, dout, dout_t, lse, lse_t, window,
                   shift=(0, 0, 0), scale=None, workspace=None, flags=0, stream=None):
    """Gradients (dq, dk, dv, dqt, dkt, dvt) of joint_attn for the output gradients
    ``dout`` (image) and ``dout_t`` (text); ``out``, ``out_t``, ``lse``, ``lse_t``
    are the forward call's outputs."""
    _check_inputs(q, k, v, out, dout)
    hkv = _kv_heads(q, k, v)
    for t in (qt, kt, vt, out_t, dout_t):
        if not isinstance(t, torch.Tensor) or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("text tensors must be torch tensors with q's dtype and device")
        if not t.is_contiguous():
            raise ValueError("text tensors must be contiguous [B, L, H, d]")
    for l_ in (lse, lse_t):
        if l_ is None or l_.dtype != torch.float32 or not l_.is_contiguous():
            raise ValueError("lse and lse_t must be the forward's contiguous fp32 log-sum-exp")
    L = qt.shape[1]
    prm = make_params(q.shape, q.dtype, window, shift, (0, 0, 0), scale, flags, hkv=hkv)
    lib = _lib.load()
    need = int(lib.basa_joint_bwd_workspace_size(ctypes.byref(prm), int(L)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    grads = [torch.empty_like(x) for x in (q, k, v, qt, kt, vt)]
    with torch.cuda.device(q.device):
        _lib.check(lib.basa_joint_attn_bwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(qt), _ptr(kt), _ptr(vt), int(L), _ptr(out),
            _ptr(out_t), _ptr(dout), _ptr(dout_t), _ptr(lse), _ptr(lse_t),
            *(_ptr(g_) for g_ in grads), _ptr(workspace), ctypes.byref(prm),
            _stream(q, stream)), "basa_joint_attn_bwd")
    return tuple(grads)


def get_status(stream=None) -> int:
    """Synchronise and return (and clear) the device status code (test use)."""
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(_lib.load().basa_get_status(ctypes.c_void_p(s.cuda_stream)))


def window_tiles(grid, window, shift=(0, 0, 0), d=128, flags=0):
    """Host-only tile plan of the bf16 kernel: int32 array [windows, tiles, 128] of
    flattened token indices per shared-memory row (-1 = padding)."""
    import numpy as np
    T, Hg, Wg = grid
    prm = make_params((1, T, Hg, Wg, 1, d), BASA_BF16, window, shift, flags=flags)
    lib = _lib.load()
    nw, nt = ctypes.c_int32(), ctypes.c_int32()
    _lib.check(lib.basa_window_tiles(ctypes.byref(prm), ctypes.byref(nw), ctypes.byref(nt),
                                     None, 0), "basa_window_tiles")
    rows = np.empty((nw.value, nt.value, 128), dtype=np.int32)
    _lib.check(lib.basa_window_tiles(ctypes.byref(prm), None, None,
                                     rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                     rows.size), "basa_window_tiles")
    return rows
