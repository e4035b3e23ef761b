"""The bounded-wait path of the tensor-core kernel, exercised without a fault.

With the test-only flag BASA_FLAG_TEST_WITHHOLD_LOADS the kernel's loader issues
no copies, so the MMA warp's first wait (for a query tile that never arrives)
runs out after the call's short time limit.  The kernel must then leave every
role loop, free its tensor memory and return; the host reads BASA_ERR_TIMEOUT
from the device status word, and the same CUDA context must keep working.
"""
import numpy as np
import pytest
import torch

import oracle
from basa_synth import make_qkv
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


def test_withheld_loads_time_out_and_context_survives(basa):
    from sparse_attention_diffusion_basa_b200._lib import BASA_FLAG_TEST_WITHHOLD_LOADS
    shape, window, shift = (1, 1, 32, 32, 2, 128), (1, 16, 16), (0, 8, 8)
    q, k, v = make_qkv(shape, "bf16", 71, 72, 73)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    assert basa.get_status() == 0
    basa.window_attn(dq, dk, dv, window, shift, flags=BASA_FLAG_TEST_WITHHOLD_LOADS,
                     wait_timeout_ms=100)
    assert basa.get_status() == 7  # BASA_ERR_TIMEOUT, and the status word is cleared
    assert basa.get_status() == 0
    out = basa.window_attn(dq, dk, dv, window, shift)
    torch.cuda.synchronize()
    ref = oracle.window_attn(oracle.as_f64(q), oracle.as_f64(k), oracle.as_f64(v),
                             oracle_params(shape, window, shift))
    assert_close(out, ref, "bf16", "after timeout")
    assert basa.get_status() == 0
