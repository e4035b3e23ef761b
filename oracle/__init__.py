"""CPU fp64 oracle for shifted local window attention (test infrastructure).

Only the tests, the package's smoke check and the benchmark's CPU-baseline leg
import this package.  It shares no code with the CUDA library: the C oracle in
``basa_oracle.c`` is compiled on its own by ``build.py`` and loaded here with
ctypes, and ``brute.py`` is an independent dense-mask restatement for tiny grids.
"""
from .oracle import (OracleParams, build_oracle, window_attn, full_attn, pool_kv,
                     joint_attn, joint_attn_bwd, window_attn_bwd, max_threads, as_f64)
from .brute import brute_window_attn, brute_joint_attn, window_ids

__all__ = ["OracleParams", "build_oracle", "window_attn", "full_attn", "pool_kv",
           "joint_attn", "joint_attn_bwd", "window_attn_bwd", "max_threads", "as_f64", "brute_window_attn", "brute_joint_attn",
           "window_ids"]
