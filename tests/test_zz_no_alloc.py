"""The allocation-free layer entry point (w4a4_linear_noalloc) against the
regular one (w4a4_linear with a caller-provided workspace).

w4a4_linear_noalloc exists for callers that cannot allocate device memory
(a program whose device memory is all in its own pool, a plugin in a runtime
that forbids cudaMalloc after start-up); it runs the same kernels on a fixed
scratch array inside the library.  This file is collected last so that a run
stopping at the first failure has already run every other test; it passes on
its own in a fresh process as well."""
from __future__ import annotations

import numpy as np
import pytest

import w4a4_int4_quantized_b200 as w4
from w4a4_int4_quantized_b200 import inputs

from gpu_util import check_output, dev_bf16, host_f64

pytestmark = pytest.mark.gpu


def _layer(seed, M, K, N, g, r):
    spec = inputs.LayerSpec("noalloc", M, K, N, g, rank=r, bias=True, seed=seed, outlier_scale=100.0)
    d = inputs.make_layer(spec)
    X, W = dev_bf16(d["X"]), dev_bf16(d["W"])
    L1 = dev_bf16(d["L1"]) if r else None
    L2 = dev_bf16(d["L2"]) if r else None
    return X, W, L1, L2, dev_bf16(d["bias"])


def test_noalloc_matches_linear_on_two_calls_in_a_row():
    import torch
    from w4a4_int4_quantized_b200 import build
    build.build()
    w4.load_library()
    results = []
    # layers back to back on the shared scratch, each checked against
    # w4a4_linear: a large one that fills most of the scratch, a smaller one
    # whose codes, scales and T sit at other offsets over that data, then one
    # larger than the second with yet another geometry, so every region a call
    # reads was last written by a different layer (stale bytes would show)
    layers = [(10, (1536, 3072, 1024, 128, 64)), (11, (640, 3072, 1024, 128, 0)),
              (12, (200, 1280, 520, 64, 32)), (13, (1000, 2048, 264, 64, 48))]
    for seed, (M, K, N, g, r) in layers:
        X, W, L1, L2, b = _layer(seed, M, K, N, g, r)
        Wq, ws = w4.w4a4_quantize_weights(W, g)
        ref = w4.w4a4_linear(X, Wq, ws, g, L1, L2, b)
        got = w4.w4a4_linear_noalloc(X, Wq, ws, g, L1, L2, b)
        torch.cuda.synchronize()
        results.append((got, ref, r))
    for got, ref, r in results:
        check_output(host_f64(got), host_f64(ref), lowrank=r > 0)
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    assert w4.w4a4_get_device_error() == 0


def test_noalloc_rejects_layers_beyond_the_scratch():
    import torch
    w4.load_library()
    M, K, N = 4608, 12288, 256          # 28.3 MB of codes > 16 MiB of scratch
    assert w4.w4a4_workspace_bytes(M, K, 0) > w4.NOALLOC_SCRATCH_BYTES
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    ws = torch.zeros((N,), dtype=torch.float32, device="cuda")
    with pytest.raises(w4.W4A4Error) as e:
        w4.w4a4_linear_noalloc(X, Wq, ws, 128)
    assert e.value.status == 7      # W4A4_ERR_WORKSPACE
