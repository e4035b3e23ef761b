"""ctypes front end of the C fp64 oracle (test infrastructure only).

Every function takes and returns float64 numpy arrays in the token layout
``[B, T, Hg, Wg, H, d]``.  Inputs stored in bf16 or fp32 are widened exactly to
float64 by ``as_f64`` before they reach the oracle.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional, Sequence, Tuple

import numpy as np

from . import build as _build


class _CParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("B", "H", "T", "Hg", "Wg", "d", "wt", "wh", "ww", "st", "sh", "sw",
                 "pt", "ph", "pw")] + [("scale", ctypes.c_double), ("Hkv", ctypes.c_int64),
                                       ("pad", ctypes.c_int64)]


@dataclass
class OracleParams:
    """Sizes of one call.  ``window``/``shift``/``pool`` are (t, rows, columns)."""

    B: int
    T: int
    Hg: int
    Wg: int
    H: int
    d: int
    window: Tuple[int, int, int]
    shift: Tuple[int, int, int] = (0, 0, 0)
    pool: Tuple[int, int, int] = (0, 0, 0)
    scale: Optional[float] = None
    Hkv: int = 0  # K/V heads (grouped-query attention); 0 = H
    pad: bool = False  # pad axes the window does not divide; padding is no token

    def c(self) -> _CParams:
        sc = self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)
        return _CParams(self.B, self.H, self.T, self.Hg, self.Wg, self.d,
                        *self.window, *self.shift, *self.pool, sc, self.Hkv, int(self.pad))

    @property
    def kv_heads(self) -> int:
        return self.Hkv if self.Hkv > 0 else self.H

    @property
    def N(self) -> int:
        return self.T * self.Hg * self.Wg

    @property
    def P(self) -> int:
        if tuple(self.pool) == (0, 0, 0):
            return 0
        return (self.T // self.pool[0]) * (self.Hg // self.pool[1]) * (self.Wg // self.pool[2])


_lib = None


def build_oracle(force: bool = False) -> str:
    return _build.build(force=force)


def _bind(path):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_pool.argtypes = [dp, dp, ctypes.POINTER(_CParams)]
    lib.oracle_pool.restype = None
    lib.oracle_window_attn.argtypes = [dp, dp, dp, dp, dp, dp, dp,
                                       ctypes.POINTER(_CParams),
                                       ctypes.POINTER(ctypes.c_int64),
                                       ctypes.c_int64, ctypes.c_int]
    lib.oracle_window_attn.restype = ctypes.c_int
    lib.oracle_window_attn_extra.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int64, dp, dp,
                                             ctypes.POINTER(_CParams),
                                             ctypes.POINTER(ctypes.c_int64),
                                             ctypes.c_int64, ctypes.c_int]
    lib.oracle_window_attn_extra.restype = ctypes.c_int
    lib.oracle_joint_text_attn.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int64, dp, dp,
                                           ctypes.POINTER(_CParams), ctypes.c_int]
    lib.oracle_joint_text_attn.restype = ctypes.c_int
    lib.oracle_window_attn_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, ctypes.POINTER(_CParams)]
    lib.oracle_joint_attn_bwd.argtypes = [dp, dp, dp, dp, dp, dp, ctypes.c_int64, dp, dp,
                                          dp, dp, dp, dp, dp, dp, ctypes.POINTER(_CParams)]
    lib.oracle_joint_attn_bwd.restype = ctypes.c_int
    lib.oracle_window_attn_bwd.restype = ctypes.c_int
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(_build.build())
    return _lib


class use_library:
    """Context manager that routes oracle calls to another compiled copy of the
    oracle (used by the tests that plant mistakes in a copy of the C source)."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _load()
        _lib = _bind(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def as_f64(x) -> np.ndarray:
    """Exact float64 copy of a torch tensor (any float dtype) or numpy array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def pool_kv(x: np.ndarray, prm: OracleParams) -> np.ndarray:
    """Mean of x over pooled cells -> [B, T/pt, Hg/ph, Wg/pw, H, d]."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    pt, ph, pw = prm.pool
    out = np.empty((prm.B, prm.T // pt, prm.Hg // ph, prm.Wg // pw, prm.kv_heads, prm.d))
    c = prm.c()
    _load().oracle_pool(_ptr(x), _ptr(out), ctypes.byref(c))
    return out


def window_attn(q, k, v, prm: OracleParams, kp=None, vp=None, want_lse=False,
                select: Optional[np.ndarray] = None, threads: int = 0):
    """Shifted-window attention.

    If ``prm.pool`` is non-zero and kp/vp are not given, they are pooled here
    from k and v.  ``select`` is an int64 array of (b, n, h) rows; then the
    result holds one output row per selected query.
    Returns ``out`` or ``(out, lse)``.
    """
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    if tuple(prm.pool) != (0, 0, 0) and kp is None:
        kp = pool_kv(k, prm)
        vp = pool_kv(v, prm)
    if kp is not None:
        kp = np.ascontiguousarray(kp, dtype=np.float64)
        vp = np.ascontiguousarray(vp, dtype=np.float64)
        if tuple(prm.pool) == (0, 0, 0):
            raise ValueError("pooled tensors given but pool is (0, 0, 0)")
    sel_ptr, nsel = None, 0
    if select is not None:
        select = np.ascontiguousarray(select, dtype=np.int64).reshape(-1, 3)
        sel_ptr = select.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
        nsel = select.shape[0]
        out = np.empty((nsel, prm.d))
        lse = np.empty((nsel,)) if want_lse else None
    else:
        out = np.empty(q.shape)
        lse = np.empty((prm.B, prm.H, prm.N)) if want_lse else None
    c = prm.c()
    rc = _load().oracle_window_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(kp), _ptr(vp),
                                    _ptr(out), _ptr(lse), ctypes.byref(c), sel_ptr,
                                    nsel, int(threads))
    if rc != 0:
        raise ValueError("oracle: window size does not divide the grid")
    return (out, lse) if want_lse else out


def full_attn(q, k, v, prm: OracleParams, want_lse=False,
              select: Optional[np.ndarray] = None, threads: int = 0):
    """Full softmax attention: one window covering the whole grid, no shift."""
    full = OracleParams(prm.B, prm.T, prm.Hg, prm.Wg, prm.H, prm.d,
                        (prm.T, prm.Hg, prm.Wg), (0, 0, 0), (0, 0, 0), prm.scale, prm.Hkv)
    return window_attn(q, k, v, full, want_lse=want_lse, select=select, threads=threads)


def joint_attn(q, k, v, qt, kt, vt, prm: OracleParams, want_lse=False,
               select: Optional[np.ndarray] = None, threads: int = 0):
    """Joint text + image attention with shifted windows for the image queries.

    Image queries (``q``, ``[B, T, Hg, Wg, H, d]``) attend to their own shifted
    window plus every text token; text queries (``qt``, ``[B, L, H, d]``) attend to
    every image token and every text token; one softmax per query.  ``prm.pool``
    must be (0, 0, 0): the text tokens take the place of the global memory.
    ``select`` (rows (b, n, h)) restricts the image outputs as in window_attn;
    the text outputs are always complete.
    Returns ``(out, out_t)`` or ``(out, out_t, lse, lse_t)``.
    """
    if tuple(prm.pool) != (0, 0, 0):
        raise ValueError("joint attention takes no pooled memory")
    q, k, v, qt, kt, vt = (np.ascontiguousarray(x, dtype=np.float64)
                           for x in (q, k, v, qt, kt, vt))
    L = qt.shape[1]
    assert qt.shape == (prm.B, L, prm.H, prm.d)
    assert kt.shape == (prm.B, L, prm.kv_heads, prm.d) and vt.shape == kt.shape
    sel_ptr, nsel = None, 0
    if select is not None:
        select = np.ascontiguousarray(select, dtype=np.int64).reshape(-1, 3)
        sel_ptr = select.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
        nsel = select.shape[0]
        out = np.empty((nsel, prm.d))
        lse = np.empty((nsel,)) if want_lse else None
    else:
        out = np.empty(q.shape)
        lse = np.empty((prm.B, prm.H, prm.N)) if want_lse else None
    c = prm.c()
    lib = _load()
    rc = lib.oracle_window_attn_extra(_ptr(q), _ptr(k), _ptr(v), _ptr(kt) if L else None,
                                      _ptr(vt) if L else None, L, _ptr(out), _ptr(lse),
                                      ctypes.byref(c), sel_ptr, nsel, int(threads))
    if rc != 0:
        raise ValueError("oracle: window size does not divide the grid")
    out_t = np.empty(qt.shape)
    lse_t = np.empty((prm.B, prm.H, L)) if want_lse else None
    rc = lib.oracle_joint_text_attn(_ptr(qt), _ptr(kt), _ptr(vt), _ptr(k), _ptr(v), L,
                                    _ptr(out_t), _ptr(lse_t), ctypes.byref(c), int(threads))
    if rc != 0:
        raise ValueError("oracle: bad text length")
    return (out, out_t, lse, lse_t) if want_lse else (out, out_t)


def joint_attn_bwd(q, k, v, qt, kt, vt, dout, dout_t, prm: OracleParams):
    """Gradients (dq, dk, dv, dqt, dkt, dvt) of joint text + image attention for
    the output gradients ``dout`` (image queries) and ``dout_t`` (text queries);
    the forward is recomputed from the inputs."""
    if tuple(prm.pool) != (0, 0, 0):
        raise ValueError("joint attention takes no pooled memory")
    q, k, v, qt, kt, vt, dout, dout_t = (np.ascontiguousarray(x, dtype=np.float64)
                                         for x in (q, k, v, qt, kt, vt, dout, dout_t))
    L = qt.shape[1]
    grads = [np.empty(x.shape) for x in (q, k, v, qt, kt, vt)]
    c = prm.c()
    rc = _load().oracle_joint_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(qt), _ptr(kt), _ptr(vt),
                                       ctypes.c_int64(L), _ptr(dout), _ptr(dout_t),
                                       *(_ptr(g) for g in grads), ctypes.byref(c))
    if rc != 0:
        raise ValueError("oracle: window size does not divide the grid")
    return tuple(grads)


def window_attn_bwd(q, k, v, dout, prm: OracleParams):
    """Gradients (dq, dk, dv) of window attention for the output gradient
    ``dout``, with the pooled global memory of ``prm.pool`` when it is set; the
    forward is recomputed from q, k, v."""
    q, k, v, dout = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, dout))
    dq, dk, dv = np.empty(q.shape), np.empty(k.shape), np.empty(v.shape)
    c = prm.c()
    rc = _load().oracle_window_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq),
                                        _ptr(dk), _ptr(dv), ctypes.byref(c))
    if rc != 0:
        raise ValueError("oracle: window or pool cell does not divide the grid")
    return dq, dk, dv
