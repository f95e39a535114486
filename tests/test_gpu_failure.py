"""The failure path of the bounded waits, on the GPU, without faulting it.

Every mbarrier wait in the kernels gives up after a time limit, records a bit
in the library's device error word and lets the kernel finish.  The self-test
entry point runs the low-rank down-projection with its operand producer
withholding every load and a 1 ms operand-wait limit: the tensor-core
issuer's wait must run out (no copy or MMA is in flight then), the kernel
must return normally, w4a4_get_device_error must report
W4A4_ERR_DEVICE_TIMEOUT with the operand-wait bit, and the next regular call
in the same process must be unaffected (bit-equal to a call made before)."""
from __future__ import annotations

import numpy as np
import pytest

import w4a4_int4_quantized_b200 as w4
from w4a4_int4_quantized_b200 import inputs

from gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_the_library_recovers():
    import ctypes
    import torch
    from w4a4_int4_quantized_b200 import build
    build.build()
    lib = w4.load_library()
    M, K, r = 300, 3072, 64
    spec = inputs.LayerSpec("timeout", M, K, 256, 128, rank=r, seed=41, outlier_scale=100.0)
    d = inputs.make_layer(spec)
    X, L1 = dev_bf16(d["X"]), dev_bf16(d["L1"])
    assert w4.w4a4_get_device_error() == 0
    _, _, T_before = w4.w4a4_rotate_quantize_act(X, 128, L1)
    torch.cuda.synchronize()

    w4.w4a4_selftest_wait_timeout(X, L1, timeout_us=1000)
    code = ctypes.c_uint(0)
    status = lib.w4a4_get_device_error(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                       ctypes.byref(code))
    assert status == 5, f"status {status}"            # W4A4_ERR_DEVICE_TIMEOUT
    assert code.value & w4.DEVERR_WAIT_OPERANDS, hex(code.value)
    assert code.value & ~(w4.DEVERR_WAIT_OPERANDS | w4.DEVERR_WAIT_SLOT) == 0, hex(code.value)
    assert w4.w4a4_get_device_error() == 0            # read-and-clear

    # the context is intact and the next regular call is unaffected
    _, _, T_after = w4.w4a4_rotate_quantize_act(X, 128, L1)
    torch.cuda.synchronize()
    assert torch.equal(T_after.view(torch.int16), T_before.view(torch.int16))
    assert w4.w4a4_get_device_error() == 0
    assert np.isfinite(T_after.float().cpu().numpy()).all()
