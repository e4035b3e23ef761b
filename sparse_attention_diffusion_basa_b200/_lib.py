"""ctypes view of the C ABI in ``include/basa.h`` (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# BASA_LIBRARY=checked selects the build whose kernels check every box and
# output index (python -m sparse_attention_diffusion_basa_b200.build --checked).
LIB_PATH = os.path.join(HERE, "_lib", "libbasa_checked.so" if os.environ.get("BASA_LIBRARY") == "checked"
                        else "libbasa.so")

BASA_OK = 0
STATUS_NAMES = {
    0: "BASA_OK", 1: "BASA_ERR_INVALID_ARG", 2: "BASA_ERR_SHAPE", 3: "BASA_ERR_UNSUPPORTED",
    4: "BASA_ERR_ALIGN", 5: "BASA_ERR_WORKSPACE", 6: "BASA_ERR_CUDA", 7: "BASA_ERR_TIMEOUT",
    8: "BASA_ERR_SCRATCH_LIMIT", 9: "BASA_ERR_CHECK",
}
BASA_F32, BASA_BF16, BASA_FP8_E4M3 = 0, 1, 2
BASA_FLAG_TEST_WITHHOLD_LOADS = 0x1
BASA_FLAG_BWD_CUDA_CORES = 0x2
BASA_FLAG_PAD_GRID = 0x4

# Every symbol include/basa.h declares.
EXPORTS = ("basa_status_string", "basa_version", "basa_workspace_size", "basa_pool_kv",
           "basa_window_attn", "basa_window_attn_gm", "basa_full_attn", "basa_get_status",
           "basa_window_tiles", "basa_window_attn_noalloc",
           "basa_joint_attn", "basa_window_attn_bwd", "basa_bwd_workspace_size",
           "basa_joint_workspace_size", "basa_joint_attn_bwd", "basa_joint_bwd_workspace_size")


class BasaParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "T", "Hg", "Wg", "d", "wt", "wh", "ww", "st", "sh", "sw",
                 "pt", "ph", "pw")] + [
        ("scale", ctypes.c_float), ("dtype", ctypes.c_int32), ("flags", ctypes.c_uint32),
        ("wait_timeout_ms", ctypes.c_uint32), ("Hkv", ctypes.c_int32),
        ("q_descale", ctypes.c_float), ("k_descale", ctypes.c_float),
        ("v_descale", ctypes.c_float)]


class BasaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}")


_lib = None


def load():
    """Load the library; raises if it has not been built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"CUDA library {LIB_PATH} is missing; build it with "
            "`python -m sparse_attention_diffusion_basa_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp = ctypes.c_void_p
    P = ctypes.POINTER(BasaParams)
    lib.basa_status_string.argtypes = [ctypes.c_int]
    lib.basa_status_string.restype = ctypes.c_char_p
    lib.basa_version.argtypes = []
    lib.basa_version.restype = ctypes.c_int
    lib.basa_workspace_size.argtypes = [P]
    lib.basa_workspace_size.restype = ctypes.c_size_t
    lib.basa_pool_kv.argtypes = [vp, vp, vp, vp, P, vp]
    lib.basa_pool_kv.restype = ctypes.c_int
    lib.basa_window_attn.argtypes = [vp, vp, vp, vp, vp, vp, P, vp]
    lib.basa_window_attn.restype = ctypes.c_int
    lib.basa_window_attn_gm.argtypes = [vp, vp, vp, vp, vp, vp, vp, P, vp]
    lib.basa_window_attn_gm.restype = ctypes.c_int
    lib.basa_full_attn.argtypes = [vp, vp, vp, vp, vp, P, vp]
    lib.basa_full_attn.restype = ctypes.c_int
    lib.basa_joint_attn.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int64, vp, vp, vp, vp, vp, P,
                                    vp]
    lib.basa_joint_attn.restype = ctypes.c_int
    lib.basa_window_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, P, vp]
    lib.basa_window_attn_bwd.restype = ctypes.c_int
    lib.basa_bwd_workspace_size.argtypes = [P]
    lib.basa_bwd_workspace_size.restype = ctypes.c_size_t
    lib.basa_joint_workspace_size.argtypes = [P, ctypes.c_int64]
    lib.basa_joint_workspace_size.restype = ctypes.c_size_t
    lib.basa_joint_bwd_workspace_size.argtypes = [P, ctypes.c_int64]
    lib.basa_joint_bwd_workspace_size.restype = ctypes.c_size_t
    lib.basa_joint_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int64] + [vp] * 13 + [P, vp]
    lib.basa_joint_attn_bwd.restype = ctypes.c_int
    lib.basa_get_status.argtypes = [vp]
    lib.basa_get_status.restype = ctypes.c_int
    lib.basa_window_tiles.argtypes = [P, ctypes.POINTER(ctypes.c_int32),
                                      ctypes.POINTER(ctypes.c_int32),
                                      ctypes.POINTER(ctypes.c_int32), ctypes.c_int64]
    lib.basa_window_tiles.restype = ctypes.c_int
    lib.basa_window_attn_noalloc.argtypes = [vp, vp, vp, vp, vp, P, vp]
    lib.basa_window_attn_noalloc.restype = ctypes.c_int
    _lib = lib
    return lib


def check(code: int, what: str):
    if code != BASA_OK:
        raise BasaError(code, what)
