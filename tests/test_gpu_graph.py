"""The layer entry point inside a CUDA graph.

w4a4_linear is a short chain of launches with programmatic dependencies
between them (with a low-rank branch of rank <= 128: the down-projection T =
X L1, then the codes kernel beside it, then the GEMM).  Captured into a graph
and replayed on new inputs written into the captured buffers, it must give
exactly what a direct call gives on the same inputs."""
from __future__ import annotations

import pytest

import w4a4_int4_quantized_b200 as w4
from w4a4_int4_quantized_b200 import inputs

from gpu_util import dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rank", [0, 64, 128, 256])
def test_layer_replays_bit_equal_from_a_graph(rank):
    import torch
    from w4a4_int4_quantized_b200 import build
    build.build()
    w4.load_library()
    M, K, N, g = 1000, 3072, 1024, 128
    spec = inputs.LayerSpec("graph", M, K, N, g, rank=rank, bias=True, seed=60 + rank, outlier_scale=100.0)
    d = inputs.make_layer(spec)
    W, b = dev_bf16(d["W"]), dev_bf16(d["bias"])
    L1 = dev_bf16(d["L1"]) if rank else None
    L2 = dev_bf16(d["L2"]) if rank else None
    Wq, ws = w4.w4a4_quantize_weights(W, g)
    X = dev_bf16(d["X"])
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    work = torch.empty((w4.w4a4_workspace_bytes(M, K, rank),), dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        w4.w4a4_linear(X, Wq, ws, g, L1, L2, b, Y=Y, workspace=work, stream=side)   # plans, tensor maps
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        w4.w4a4_linear(X, Wq, ws, g, L1, L2, b, Y=Y, workspace=work, stream=torch.cuda.current_stream())
    for seed in (1, 2, 3):
        Xn = dev_bf16(inputs.make_activations(spec, __import__("numpy").random.default_rng(seed)))
        X.copy_(Xn)
        graph.replay()
        torch.cuda.synchronize()
        ref = w4.w4a4_linear(Xn, Wq, ws, g, L1, L2, b)
        torch.cuda.synchronize()
        assert torch.equal(Y.view(torch.int16), ref.view(torch.int16)), f"rank {rank}, seed {seed}"
    del graph
    assert w4.w4a4_get_device_error() == 0
