"""Host-side tests of the C ABI: symbols, validation codes and the window tile
plan.  None of these launch anything, so they run without a GPU."""
import ctypes
import itertools
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="session")
def lib():
    from sparse_attention_diffusion_basa_b200 import build
    build.build()
    from sparse_attention_diffusion_basa_b200 import _lib
    return _lib.load()


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "basa.h")).read()
    return sorted(set(re.findall(r"BASA_API\s+[\w\s\*]*?\b(basa_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    from sparse_attention_diffusion_basa_b200 import _lib
    declared = _declared_symbols()
    assert len(declared) >= 9
    assert set(declared) == set(_lib.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name
    assert lib.basa_version() >= 100
    for code in range(9):
        assert lib.basa_status_string(code)


def _p(**kw):
    from sparse_attention_diffusion_basa_b200 import make_params
    shape = kw.pop("shape", (1, 1, 16, 16, 2, 64))
    dtype = kw.pop("dtype", 1)
    return make_params(shape, dtype, kw.pop("window", (1, 8, 8)), kw.pop("shift", (0, 4, 4)),
                       kw.pop("pool", (0, 0, 0)), kw.pop("scale", None))


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def test_validation_codes(lib):
    from sparse_attention_diffusion_basa_b200 import _lib
    call = lambda prm, q=_fake(), ws=None: lib.basa_window_attn(
        q, _fake(), _fake(), _fake(), None, ws, ctypes.byref(prm), None)
    assert call(_p(window=(1, 5, 8))) == 2                      # does not divide the grid
    assert call(_p(window=(0, 8, 8))) == 1                      # zero window
    assert call(_p(shape=(1, 1, 16, 16, 2, 48))) == 3           # head dim
    assert call(_p(shape=(1, 1, 16, 16, 2, 32), dtype=1)) == 3  # bf16 needs d in {64, 128}
    assert call(_p(), q=_fake(0x10008)) == 4                    # misaligned
    assert call(_p(), q=None) == 1                              # null
    assert call(_p(pool=(1, 2, 2))) == 5                        # workspace missing
    assert call(_p(pool=(1, 3, 2))) == 2                        # pool does not divide
    assert call(_p(pool=(0, 2, 2))) == 1                        # partial pool spec
    prm = _p()
    prm.dtype = 7
    assert call(prm) == 1
    # empty problems are valid no-ops and touch nothing
    assert call(_p(shape=(0, 1, 16, 16, 2, 64)), q=None) == 0
    assert lib.basa_full_attn(None, None, None, None, None,
                              ctypes.byref(_p(shape=(1, 1, 16, 16, 0, 64))), None) == 0
    # bf16 plans whose wrapped boxes are not a multiple of 8 tokens are refused
    assert call(_p(shape=(1, 1, 16, 16, 2, 64), window=(1, 8, 8), shift=(0, 3, 3))) == 3
    # gm variant needs pooled tensors and a pool spec
    assert lib.basa_window_attn_gm(_fake(), _fake(), _fake(), None, None, _fake(), None,
                                   ctypes.byref(_p(pool=(1, 2, 2))), None) == 1
    assert lib.basa_window_attn_gm(_fake(), _fake(), _fake(), _fake(), _fake(), _fake(), None,
                                   ctypes.byref(_p()), None) == 1
    # pooling: needs a pool spec, aligned pointers
    assert lib.basa_pool_kv(_fake(), _fake(), _fake(), _fake(), ctypes.byref(_p()), None) == 1
    assert lib.basa_pool_kv(_fake(), _fake(), _fake(0x10004), _fake(),
                            ctypes.byref(_p(pool=(1, 2, 2))), None) == 4
    assert _lib.STATUS_NAMES[4] == "BASA_ERR_ALIGN"


def test_noalloc_refuses_problems_beyond_its_scratch(lib):
    # pooled K + V of 2 x [B, P, H, d] bf16 = 2 x 4 x 1024 x 24 x 128 x 2 bytes > 32 MiB
    prm = _p(shape=(4, 1, 128, 128, 24, 128), window=(1, 16, 16), shift=(0, 8, 8),
             pool=(1, 4, 4))
    assert lib.basa_window_attn_noalloc(_fake(), _fake(), _fake(), _fake(), None,
                                        ctypes.byref(prm), None) == 8
    assert lib.basa_status_string(8)
    # validation runs first, exactly as for basa_window_attn
    assert lib.basa_window_attn_noalloc(_fake(0x10008), _fake(), _fake(), _fake(), None,
                                        ctypes.byref(_p(pool=(1, 2, 2))), None) == 4


def test_workspace_size(lib):
    from sparse_attention_diffusion_basa_b200 import workspace_size
    import torch
    assert workspace_size((1, 1, 16, 16, 2, 64), torch.bfloat16, (1, 8, 8)) == 0
    # pooled K and V of [B, P, H, d] bf16, each rounded up to 256 bytes
    n = 2 * 64 * 24 * 128 * 2
    assert workspace_size((2, 1, 32, 32, 24, 128), torch.bfloat16, (1, 16, 16),
                          pool=(1, 4, 4)) == 2 * ((n + 255) // 256 * 256)
    assert workspace_size((1, 1, 4, 4, 1, 32), torch.float32, (1, 2, 2),
                          pool=(1, 2, 2)) == 2 * 512  # 4 cells x 32 x fp32


def _window_sets(grid, window, shift):
    """Token sets of every shifted window, from the window-id formula."""
    T, Hg, Wg = grid
    ids = {}
    for t, y, x in itertools.product(range(T), range(Hg), range(Wg)):
        key = (((t - shift[0]) % T) // window[0], ((y - shift[1]) % Hg) // window[1],
               ((x - shift[2]) % Wg) // window[2])
        ids.setdefault(key, set()).add((t * Hg + y) * Wg + x)
    return ids


PLAN_CASES = [
    ((1, 16, 16), (1, 8, 8), [(0, 0, 0), (0, 4, 0), (0, 0, 4), (0, 4, 4)]),
    ((1, 64, 64), (1, 16, 16), [(0, 0, 0), (0, 8, 8), (0, 8, 0), (0, 0, 8), (0, -8, 24)]),
    ((21, 45, 80), (7, 9, 16), [(3, 4, 8), (0, 0, 0), (1, 5, 8), (6, 8, 0)]),
    ((4, 6, 32), (2, 3, 16), [(1, 1, 8), (1, 2, 0)]),
    ((2, 8, 8), (2, 8, 8), [(0, 0, 0), (1, 0, 0)]),
    ((1, 24, 8), (1, 24, 8), [(0, 5, 0), (0, 16, 0)]),
]


@pytest.mark.parametrize("grid,window,shifts", PLAN_CASES)
def test_tile_plan_covers_each_shifted_window_once(lib, grid, window, shifts):
    from sparse_attention_diffusion_basa_b200 import window_tiles
    for shift in shifts:
        rows = window_tiles(grid, window, shift)
        sets = _window_sets(grid, window, shift)
        assert rows.shape[0] == len(sets)
        m = window[0] * window[1] * window[2]
        seen = set()
        for w in range(rows.shape[0]):
            toks = rows[w][rows[w] >= 0]
            assert len(toks) == m, (shift, w)
            assert len(set(toks.tolist())) == m
            assert set(toks.tolist()) in [s for s in sets.values()], (shift, w)
            seen |= set(toks.tolist())
            # every 128-row tile is a prefix of real rows followed by padding
            for tile in rows[w]:
                n = int((tile >= 0).sum())
                assert (tile[:n] >= 0).all() and (tile[n:] < 0).all()
                assert n % 8 == 0
        assert seen == set(range(grid[0] * grid[1] * grid[2]))


PADDED_PLAN_CASES = [  # grids the window does not divide (BASA_FLAG_PAD_GRID)
    ((1, 48, 85), (1, 16, 16), [(0, 0, 0), (0, 8, 8), (0, 8, 0)]),
    ((1, 5, 7), (1, 16, 16), [(0, 0, 0), (0, 8, 8)]),
    ((13, 18, 32), (7, 9, 16), [(3, 4, 8), (0, 0, 0)]),
    ((5, 10, 16), (3, 5, 8), [(1, 2, 0)]),
]


@pytest.mark.parametrize("grid,window,shifts", PADDED_PLAN_CASES)
def test_padded_tile_plan_holds_each_padded_window(lib, grid, window, shifts):
    """Each window's tiles hold exactly the real tokens that share its window ids
    on the padded axes (ids from the brute-force module's reading: padding at the
    far end, the shift rolling the padded axis); every token appears once."""
    from oracle import window_ids
    from sparse_attention_diffusion_basa_b200 import window_tiles, BASA_FLAG_PAD_GRID
    T, Hg, Wg = grid
    for shift in shifts:
        rows = window_tiles(grid, window, shift, flags=BASA_FLAG_PAD_GRID)
        ids = [window_ids(G, w, s, pad=True) for G, w, s in zip(grid, window, shift)]
        wid = np.stack(np.meshgrid(*ids, indexing="ij"), axis=-1).reshape(-1, 3)
        groups = {}
        for n, key in enumerate(map(tuple, wid)):
            groups.setdefault(key, set()).add(n)
        assert rows.shape[0] == np.prod([-(-G // w) for G, w in zip(grid, window)])
        seen = []
        for w in range(rows.shape[0]):
            toks = rows[w][rows[w] >= 0].tolist()
            assert len(set(toks)) == len(toks) > 0
            assert set(toks) in groups.values(), (shift, w)
            seen += toks
        assert sorted(seen) == list(range(T * Hg * Wg))


def test_tile_plan_counts(lib):
    from sparse_attention_diffusion_basa_b200 import window_tiles
    assert window_tiles((1, 128, 128), (1, 16, 16), (0, 8, 8)).shape == (64, 2, 128)
    # the video window of 7 x 9 x 16 tokens: seven 8-row tiles and one of 7 x 1 rows
    r = window_tiles((21, 45, 80), (7, 9, 16), (3, 4, 8))
    assert r.shape == (75, 8, 128)
    assert sorted(int((t >= 0).sum()) for t in r[0]) == [112] + [128] * 7


def test_tile_plan_rejects_unsupported(lib):
    from sparse_attention_diffusion_basa_b200 import window_tiles, BasaError
    with pytest.raises(BasaError):
        window_tiles((1, 16, 256), (1, 16, 256), (0, 0, 0))   # window row wider than 128
    with pytest.raises(BasaError):
        window_tiles((1, 16, 16), (1, 8, 8), (0, 3, 5))        # wrapped boxes of 3 x 5 tokens


def test_joint_and_grouped_query_validation(lib):
    """Joint attention and grouped-query K/V are validated before anything runs."""
    f = _fake
    joint = lambda prm, L=4: lib.basa_joint_attn(f(), f(), f(), f(), f(), f(), L, f(), f(), None,
                                                 None, None, ctypes.byref(prm), None)
    assert joint(_p(pool=(1, 2, 2))) == 3          # text tokens take the global-memory slot
    assert joint(_p(), L=-1) == 1                   # negative text length
    assert joint(_p(shape=(0, 1, 16, 16, 2, 64))) == 0  # empty image stream: no-op
    assert lib.basa_joint_attn(f(), f(), f(), None, f(), f(), 4, f(), f(), None, None, None,
                               ctypes.byref(_p()), None) == 1  # null text q
    assert lib.basa_joint_attn(f(), f(), f(), f(0x10008), f(), f(), 4, f(), f(), None, None,
                               None, ctypes.byref(_p()), None) == 4  # misaligned text q
    win = lambda prm: lib.basa_window_attn(f(), f(), f(), f(), None, None, ctypes.byref(prm), None)
    prm = _p(shape=(1, 1, 16, 16, 4, 64))
    prm.Hkv = 3                                     # 4 query heads are not a multiple of 3
    assert win(prm) == 1
    prm.Hkv = -1
    assert win(prm) == 1
    # pooled workspace is sized by the K/V heads
    prm = _p(shape=(1, 1, 16, 16, 4, 64), pool=(1, 2, 2))
    full = lib.basa_workspace_size(ctypes.byref(prm))
    prm.Hkv = 2
    assert lib.basa_workspace_size(ctypes.byref(prm)) * 2 == full


def test_backward_workspace_sizes(lib):
    """The backward workspace holds D = rowsum(dO * O) (fp32 [B, H, N]); with
    pooled memory also the pooled K, V (input dtype) and their fp32 gradients
    ([B, P, Hkv, d] each), every piece rounded up to 256 bytes."""
    up = lambda x: (x + 255) // 256 * 256
    B, T, Hg, Wg, H, d = 1, 1, 16, 16, 2, 64
    N = T * Hg * Wg
    plain = lib.basa_bwd_workspace_size(ctypes.byref(_p()))
    assert plain == up(B * H * N * 4)
    P = (Hg // 4) * (Wg // 4)
    for dtype, es in ((1, 2), (0, 4)):
        pooled = lib.basa_bwd_workspace_size(ctypes.byref(_p(pool=(1, 4, 4), dtype=dtype)))
        assert pooled == up(B * H * N * 4) + 2 * up(B * P * H * d * es) + 2 * up(B * P * H * d * 4)
    assert lib.basa_bwd_workspace_size(ctypes.byref(_p(pool=(1, 3, 3)))) == 0  # cell does not divide


def test_joint_workspace_needs_bf16_and_text(lib):
    """No split workspace for fp32, for L <= 0, or for invalid params; the bf16
    size depends on the device's SM count, so only its form is checked here."""
    assert lib.basa_joint_workspace_size(ctypes.byref(_p(dtype=0)), 512) == 0
    assert lib.basa_joint_workspace_size(ctypes.byref(_p()), 0) == 0
    assert lib.basa_joint_workspace_size(ctypes.byref(_p()), -3) == 0
    assert lib.basa_joint_workspace_size(ctypes.byref(_p(window=(1, 5, 5))), 64) == 0
    n = lib.basa_joint_workspace_size(ctypes.byref(_p()), 64)
    assert n % 256 == 0


def test_fp8_and_padding_validation(lib):
    """Host-side checks of e4m3 inputs and padded grids, all refused before any
    launch (fake pointers are never dereferenced)."""
    from sparse_attention_diffusion_basa_b200 import BASA_FLAG_PAD_GRID
    f8 = 2
    call = lambda prm: lib.basa_window_attn(_fake(), _fake(), _fake(), _fake(), None, None,
                                            ctypes.byref(prm), None)
    # e4m3: d = 128 only, no pooled memory, no negative or infinite descale
    assert call(_p(shape=(1, 1, 16, 16, 2, 64), dtype=f8)) == 3
    assert call(_p(shape=(1, 1, 16, 16, 2, 128), dtype=f8, pool=(1, 2, 2))) == 3
    prm = _p(shape=(1, 1, 16, 16, 2, 128), dtype=f8)
    prm.v_descale = -1.0
    assert call(prm) == 1
    prm.v_descale = float("inf")
    assert call(prm) == 1
    # e4m3 is refused by every entry point other than window and full attention
    p8 = _p(shape=(1, 1, 16, 16, 2, 128), dtype=f8)
    assert lib.basa_window_attn_gm(_fake(), _fake(), _fake(), _fake(), _fake(), _fake(), None,
                                   ctypes.byref(p8), None) == 3
    assert lib.basa_pool_kv(_fake(), _fake(), _fake(), _fake(), ctypes.byref(p8), None) == 3
    assert lib.basa_window_attn_bwd(*[_fake()] * 5, None, *[_fake()] * 3, None,
                                    ctypes.byref(p8), None) == 3
    assert lib.basa_joint_attn(*[_fake()] * 6, 4, _fake(), _fake(), None, None, None,
                               ctypes.byref(p8), None) == 3
    assert lib.basa_joint_bwd_workspace_size(ctypes.byref(p8), 4) == 0
    # padded grids: without the flag a shape error, with it the sizes follow N
    shape = (2, 1, 20, 28, 3, 64)
    assert call(_p(shape=shape, window=(1, 16, 16), shift=(0, 8, 8))) == 2
    pp = _p(shape=shape, window=(1, 16, 16), shift=(0, 8, 8))
    pp.flags = BASA_FLAG_PAD_GRID
    N = 20 * 28
    align = lambda x: (x + 255) // 256 * 256
    assert lib.basa_bwd_workspace_size(ctypes.byref(pp)) == align(2 * 3 * N * 4)
    assert lib.basa_joint_bwd_workspace_size(ctypes.byref(pp), 77) == \
        align(2 * 3 * N * 4) + align(2 * 3 * 77 * 4) + 2 * align(2 * 77 * 3 * 64 * 4)
    # the pool cell must still divide the grid
    pp.ph, pp.pw, pp.pt = 3, 4, 1
    assert call(pp) == 2
