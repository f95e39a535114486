"""GPU parity of the CUDA path (called through the C ABI) against the CPU
oracle: bit-exact codes, scales and int32 accumulators; bf16 outputs within
the stated tolerance.  Inputs are the seeded synthetic workloads."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import w4a4_int4_quantized_b200 as w4
from w4a4_int4_quantized_b200 import inputs

from gpu_util import check_output, dev_bf16, host_bits, host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from w4a4_int4_quantized_b200 import build
    build.build()
    w4.load_library()
    yield
    assert w4.w4a4_get_device_error() == 0


def _x(M, K, seed, outliers=True):
    spec = inputs.LayerSpec("t", M, K, 8, 128, seed=seed,
                            outlier_scale=100.0 if outliers else 1.0)
    return inputs.make_activations(spec, np.random.default_rng(seed))


ACT_CASES = [
    # (M, K, group)
    (64, 256, 64),
    (303, 3072, 128),
    (37, 12288, 128),
    (17, 384, 0),
    (1, 128, 64),
    (3, 16384, 64),
    (2, 32768, 128),
    (129, 1024, 64),
]


@pytest.mark.parametrize("M,K,g", ACT_CASES)
def test_act_quant_int4_bitexact(M, K, g):
    X = _x(M, K, seed=M + K + g)
    Xq, xs, _ = w4.w4a4_rotate_quantize_act(dev_bf16(X), g)
    ref_p, ref_s, _ = oracle.quantize_w4(X, g)
    got_p = Xq.cpu().numpy()
    assert np.array_equal(xs.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    assert np.array_equal(got_p, ref_p), f"{np.count_nonzero(got_p != ref_p)} code bytes differ"


@pytest.mark.parametrize("M,K,g", ACT_CASES[:5])
def test_act_quant_int8_bitexact(M, K, g):
    X = _x(M, K, seed=7 * M + K + g)
    Xq, xs = w4.w8a8_rotate_quantize_act(dev_bf16(X), g)
    ref_q, ref_s = oracle.quantize_w8(X, g)
    assert np.array_equal(xs.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    assert np.array_equal(Xq.cpu().numpy(), ref_q)


def _pad_row(vals, K):
    row = np.zeros(K, dtype=np.float32)
    row[: len(vals)] = vals
    return row


def test_ties_and_special_rows():
    """Exact half-way quotients must round to even (the slow path of the
    kernel); zero rows give scale 0 and zero codes; one-hot and constant
    groups hit the closed forms."""
    K = 256
    rows = [
        _pad_row([7, 2.5, -2.5, 3.5, -3.5, 0.5, -0.5, 1.5], K),
        _pad_row([14, 5, 3, -3, 1, -7], K),
        _pad_row([-3.5, 1.25, 0.25, -0.75], K),
        np.zeros(K, dtype=np.float32),
        np.full(K, -0.0, dtype=np.float32),
        np.full(K, 0.75, dtype=np.float32),
        _pad_row([0] * 37 + [5.0], K),
    ]
    X = inputs.f32_to_bf16_bits(np.stack(rows))
    for g in (0, 64, 128):
        Xq, xs, _ = w4.w4a4_rotate_quantize_act(dev_bf16(X), g)
        ref_p, ref_s, _ = oracle.quantize_w4(X, g)
        assert np.array_equal(xs.cpu().numpy(), ref_s)
        assert np.array_equal(Xq.cpu().numpy(), ref_p), g
    rows8 = [_pad_row([127, 0.5, 1.5, 2.5, -126.5, -3.5], K), _pad_row([-254, 1, 3, 5], K)]
    X8 = inputs.f32_to_bf16_bits(np.stack(rows8))
    Xq8, xs8 = w4.w8a8_rotate_quantize_act(dev_bf16(X8), 0)
    ref_q8, ref_s8 = oracle.quantize_w8(X8, 0)
    assert np.array_equal(Xq8.cpu().numpy(), ref_q8)
    assert np.array_equal(xs8.cpu().numpy(), ref_s8)


def test_weight_quant_bitexact():
    W = inputs.random_bf16((264, 640), seed=3, std=0.02)
    for g in (64, 128, 0):
        Wq, ws = w4.w4a4_quantize_weights(dev_bf16(W), g)
        ref_p, ref_s, _ = oracle.quantize_w4(W, g)
        assert np.array_equal(Wq.cpu().numpy(), ref_p)
        assert np.array_equal(ws.cpu().numpy(), ref_s)


GEMM_CASES = [
    # (M, N, K, group, rank, bias)
    (64, 256, 256, 64, 16, False),      # the tiny workload
    (200, 264, 384, 128, 0, True),      # ragged M and N tiles
    (1, 8, 128, 0, 0, True),            # smallest shapes, rotation off
    (130, 520, 1280, 64, 32, True),
    (257, 768, 3072, 128, 0, True),
    (96, 512, 12288, 128, 128, False),  # long K
    (300, 640, 1024, 64, 144, False),   # two low-rank chunks, the second 16 ranks
    (2048, 3072, 256, 128, 256, True),  # rank 256 and more tiles than pairs: buffer hand-off across tiles
    (512, 3072, 3072, 128, 0, True),    # few tiles: split-K over two pairs per tile
    (256, 1024, 12288, 64, 0, False),   # split-K over four pairs per tile, long K
    (1, 3072, 3072, 128, 0, True),      # split-K with a single token row
    (40, 8, 3072, 128, 0, False),       # split-K, one tile holding 8 of its 256 columns
    (256, 1024, 12288, 128, 32, True),  # split-K with the low-rank term in the reduction
    (130, 520, 12288, 128, 16, True),   # the same with ragged M and N: zero-filled T rows and L2 columns
    (3, 264, 6144, 128, 32, True),      # the same at three token rows
]


def _layer(M, N, K, g, r, bias, seed):
    spec = inputs.LayerSpec("g", M, K, N, g, rank=r, bias=bias, seed=seed, outlier_scale=100.0)
    return inputs.make_layer(spec)


@pytest.mark.parametrize("M,N,K,g,r,bias", GEMM_CASES)
def test_w4a4_layer_parity(M, N, K, g, r, bias):
    import torch
    d = _layer(M, N, K, g, r, bias, seed=M * 3 + N + K + r)
    ref = oracle.linear_w4a4(d["X"], d["W"], g, d["L1"], d["L2"], d["bias"])
    X, W = dev_bf16(d["X"]), dev_bf16(d["W"])
    L1 = dev_bf16(d["L1"]) if r else None
    L2 = dev_bf16(d["L2"]) if r else None
    b = dev_bf16(d["bias"]) if bias else None
    Wq, ws = w4.w4a4_quantize_weights(W, g)
    Xq, xs, T = w4.w4a4_rotate_quantize_act(X, g, L1)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    Y = w4.w4a4_gemm(Xq, xs, Wq, ws, g, T, L2, b, acc_debug=acc)
    torch.cuda.synchronize()
    assert np.array_equal(Wq.cpu().numpy(), ref["w_packed"])
    assert np.array_equal(Xq.cpu().numpy(), ref["x_packed"])
    got_acc = acc.cpu().numpy()
    assert np.array_equal(got_acc, ref["acc"]), f"{np.count_nonzero(got_acc != ref['acc'])} accumulators differ"
    if r:
        t_ref = ref["T"]
        assert np.max(np.abs(host_f64(T) - t_ref)) <= 1e-2 * np.max(np.abs(t_ref))
    check_output(host_f64(Y), ref["Y"], lowrank=r > 0)
    # the fused whole-layer call gives the same bits as the two-step path
    Y2 = w4.w4a4_linear(X, Wq, ws, g, L1, L2, b)
    torch.cuda.synchronize()
    assert torch.equal(Y2.view(torch.int16), Y.view(torch.int16))


@pytest.mark.parametrize("M,N,K,g", [(64, 256, 256, 128), (200, 264, 384, 128), (2, 3072, 256, 128),
                                     (257, 520, 3072, 0)])
def test_w8a8_layer_parity(M, N, K, g):
    import torch
    d = _layer(M, N, K, g, 0, True, seed=M + N + K + 1)
    ref = oracle.linear_w8a8(d["X"], d["W"], g, d["bias"])
    X, W, b = dev_bf16(d["X"]), dev_bf16(d["W"]), dev_bf16(d["bias"])
    Wq, ws = w4.w8a8_quantize_weights(W, g)
    Xq, xs = w4.w8a8_rotate_quantize_act(X, g)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    Y = w4.w8a8_gemm(Xq, xs, Wq, ws, g, b, acc_debug=acc)
    torch.cuda.synchronize()
    assert np.array_equal(Wq.cpu().numpy(), ref["w_q"])
    assert np.array_equal(Xq.cpu().numpy(), ref["x_q"])
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    check_output(host_f64(Y), ref["Y"], lowrank=False)
    Y2 = w4.w8a8_linear(X, Wq, ws, g, b)
    torch.cuda.synchronize()
    assert torch.equal(Y2.view(torch.int16), Y.view(torch.int16))


@pytest.mark.parametrize("N,K,g", [(264, 640, 64), (264, 640, 128), (264, 640, 0), (40, 12288, 128),
                                   (3072, 3072, 128)])
def test_w4a8_weight_quant_bitexact(N, K, g):
    """Asymmetric 4-bit weights with a zero point: packed codes, scale bits
    and zero points identical to the oracle (rows with outlier channels make
    the minimum and maximum sit far apart)."""
    W = inputs.random_bf16((N, K), seed=N + K + g, std=0.02)
    W[:, 5] = inputs.f32_to_bf16_bits(inputs.bf16_bits_to_f32(W[:, 5]) * 60.0)
    Wq, ws, wz = w4.w4a8_quantize_weights(dev_bf16(W), g)
    ref_p, ref_s, ref_z, _ = oracle.quantize_w4a8_weights(W, g)
    assert np.array_equal(ws.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    assert np.array_equal(wz.cpu().numpy(), ref_z)
    got = Wq.cpu().numpy()
    assert np.array_equal(got, ref_p), f"{np.count_nonzero(got != ref_p)} code bytes differ"


def test_w4a8_weight_quant_special_rows():
    """A constant row (s = 0, z = 0, codes 0), an all-positive row (zero point
    clamped to 0) and an all-negative row (clamped to 15)."""
    K = 256
    rows = np.stack([np.full(K, 0.5, np.float32),
                     np.linspace(1.0, 3.0, K, dtype=np.float32),
                     -np.linspace(1.0, 3.0, K, dtype=np.float32),
                     np.zeros(K, np.float32)])
    W = inputs.f32_to_bf16_bits(rows)
    for g in (0, 64):
        Wq, ws, wz = w4.w4a8_quantize_weights(dev_bf16(W), g)
        ref_p, ref_s, ref_z, _ = oracle.quantize_w4a8_weights(W, g)
        assert np.array_equal(ws.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
        assert np.array_equal(wz.cpu().numpy(), ref_z)
        assert np.array_equal(Wq.cpu().numpy(), ref_p)


@pytest.mark.parametrize("M,N,K,g", [(64, 256, 256, 128), (200, 264, 384, 64), (2, 3072, 256, 128),
                                     (257, 520, 3072, 0), (300, 768, 12288, 128),
                                     (3, 264, 6144, 128)])   # split-K at three token rows, ragged N
def test_w4a8_layer_parity(M, N, K, g):
    import torch
    d = _layer(M, N, K, g, 0, True, seed=M + N + K + 2)
    ref = oracle.linear_w4a8(d["X"], d["W"], g, d["bias"])
    X, W, b = dev_bf16(d["X"]), dev_bf16(d["W"]), dev_bf16(d["bias"])
    Wq, ws, wz = w4.w4a8_quantize_weights(W, g)
    Xq, xs = w4.w8a8_rotate_quantize_act(X, g)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    Y = w4.w4a8_gemm(Xq, xs, Wq, ws, wz, g, b, acc_debug=acc)
    torch.cuda.synchronize()
    assert np.array_equal(Wq.cpu().numpy(), ref["w_packed"])
    assert np.array_equal(wz.cpu().numpy(), ref["w_zero"])
    assert np.array_equal(Xq.cpu().numpy(), ref["x_q"])
    got = acc.cpu().numpy()
    assert np.array_equal(got, ref["acc"]), f"{np.count_nonzero(got != ref['acc'])} accumulators differ"
    check_output(host_f64(Y), ref["Y"], lowrank=False)
    Y2 = w4.w4a8_linear(X, Wq, ws, wz, g, b)
    torch.cuda.synchronize()
    assert torch.equal(Y2.view(torch.int16), Y.view(torch.int16))


@pytest.mark.parametrize("r,rl,scale", [(0, 32, 1.0), (16, 32, 0.3), (64, 64, 1.7)])
def test_lora_merge_bitexact(r, rl, scale):
    import torch
    K, N = 640, 264
    L1 = inputs.random_bf16((K, r), seed=1, std=0.05) if r else None
    L2 = inputs.random_bf16((r, N), seed=2, std=0.05) if r else None
    A = inputs.random_bf16((K, rl), seed=3, std=0.05)
    B = inputs.random_bf16((rl, N), seed=4, std=0.05)
    L1o, L2o = w4.w4a4_lora_merge(dev_bf16(L1) if r else None, dev_bf16(L2) if r else None,
                                  dev_bf16(A), dev_bf16(B), scale)
    ref1, ref2 = oracle.lora_merge(L1, L2, A, B, scale)
    assert np.array_equal(L1o.cpu().view(torch.int16).numpy().view(np.uint16), ref1)
    assert np.array_equal(L2o.cpu().view(torch.int16).numpy().view(np.uint16), ref2)


@pytest.mark.parametrize("M,N,K,g,r,rl,scale", [(130, 520, 1280, 64, 32, 16, 0.7), (257, 768, 3072, 128, 0, 64, 1.0),
                                                 (96, 512, 12288, 128, 128, 128, 0.25)])
def test_w4a4_layer_with_runtime_lora(M, N, K, g, r, rl, scale):
    """The merged operands in the unchanged W4A4 path give the layer with the
    LoRA beside the SVDQuant branch (oracle: unmerged, fp64)."""
    import torch
    d = _layer(M, N, K, g, r, True, seed=M + N + K + rl)
    A = inputs.random_bf16((K, rl), seed=M + 5, std=0.01)
    B = inputs.random_bf16((rl, N), seed=N + 6, std=0.01)
    ref = oracle.linear_w4a4_lora(d["X"], d["W"], g, d["L1"], d["L2"], A, B, scale, d["bias"])
    X, W, b = dev_bf16(d["X"]), dev_bf16(d["W"]), dev_bf16(d["bias"])
    Wq, ws = w4.w4a4_quantize_weights(W, g)
    L1m, L2m = w4.w4a4_lora_merge(dev_bf16(d["L1"]) if r else None, dev_bf16(d["L2"]) if r else None,
                                  dev_bf16(A), dev_bf16(B), scale)
    Y = w4.w4a4_linear(X, Wq, ws, g, L1m, L2m, b)
    torch.cuda.synchronize()
    check_output(host_f64(Y), ref["Y"], lowrank=True)


@pytest.mark.parametrize("M,N,K,g,r", [(130, 520, 1280, 64, 32), (257, 768, 3072, 128, 0),
                                     (256, 1024, 12288, 128, 32),    # split-K, low-rank term in the reduction
                                     (5, 264, 6144, 128, 16)])       # the same at five token rows, ragged N
def test_w4a4_layer_with_fused_gelu(M, N, K, g, r):
    """GELU(tanh) fused into the epilogue: the same accumulators, GELU of the
    unrounded output within the layer tolerance, and the fused call equal to
    the two-step path."""
    import torch
    d = _layer(M, N, K, g, r, True, seed=M + N + K + 9)
    ref = oracle.linear_w4a4_gelu(d["X"], d["W"], g, d["L1"], d["L2"], d["bias"])
    X, W, b = dev_bf16(d["X"]), dev_bf16(d["W"]), dev_bf16(d["bias"])
    L1 = dev_bf16(d["L1"]) if r else None
    L2 = dev_bf16(d["L2"]) if r else None
    Wq, ws = w4.w4a4_quantize_weights(W, g)
    Xq, xs, T = w4.w4a4_rotate_quantize_act(X, g, L1)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    Y = w4.w4a4_gemm_gelu(Xq, xs, Wq, ws, g, T, L2, b, acc_debug=acc)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    check_output(host_f64(Y), ref["Y"], lowrank=r > 0)
    Y2 = w4.w4a4_linear_gelu(X, Wq, ws, g, L1, L2, b)
    torch.cuda.synchronize()
    assert torch.equal(Y2.view(torch.int16), Y.view(torch.int16))


@pytest.mark.parametrize("K,act", [(3072, False), (3072, True), (12288, False)])
def test_split_k_equals_the_persistent_form(K, act):
    """A layer with few tiles runs in the split-K form (its K range spread
    over a cluster of pairs, int32 partials summed through distributed shared
    memory).  Quantization is per token, so the first 256 rows of a large
    layer (many tiles: the persistent form) must come out bit for bit the
    same as those rows run on their own."""
    import torch
    M, N, g = 4608, 3072, 128
    d = _layer(M, N, K, g, 0, True, seed=K + (7 if act else 3))
    X, W, b = dev_bf16(d["X"]), dev_bf16(d["W"]), dev_bf16(d["bias"])
    Wq, ws = w4.w4a4_quantize_weights(W, g)
    lin = w4.w4a4_linear_gelu if act else w4.w4a4_linear
    Y_all = lin(X, Wq, ws, g, None, None, b)
    Y_few = lin(X[:256].contiguous(), Wq, ws, g, None, None, b)
    torch.cuda.synchronize()
    assert torch.equal(Y_few.view(torch.int16), Y_all[:256].view(torch.int16))


def test_split_k_w4a8_equals_the_persistent_form():
    """The W4A8 GEMM's split-K form: the first 256 rows of a 4608-row layer
    bit for bit the same as those rows run on their own."""
    import torch
    M, N, K, g = 4608, 3072, 12288, 128
    d = _layer(M, N, K, g, 0, True, seed=77)
    X, W, b = dev_bf16(d["X"]), dev_bf16(d["W"]), dev_bf16(d["bias"])
    Wq, ws, wz = w4.w4a8_quantize_weights(W, g)
    Y_all = w4.w4a8_linear(X, Wq, ws, wz, g, b)
    Y_few = w4.w4a8_linear(X[:256].contiguous(), Wq, ws, wz, g, b)
    torch.cuda.synchronize()
    assert torch.equal(Y_few.view(torch.int16), Y_all[:256].view(torch.int16))


def test_fused_mlp_chain():
    """w4a4_mlp = down(gelu(up(X))): its activated tensor is the fused
    up-projection (checked against the fp64 oracle), and its output equals the
    down-projection layer applied to that tensor (bit for bit), which in turn
    matches the oracle fed the same bf16 tensor."""
    import torch
    M, D, H, g, r = 200, 512, 1536, 128, 32
    rng = np.random.default_rng(77)
    spec_up = inputs.LayerSpec("up", M, D, H, g, rank=r, bias=True, seed=78, outlier_scale=50.0)
    du = inputs.make_layer(spec_up)
    Wd = inputs.random_bf16((D, H), seed=79, std=0.02)
    L1d = inputs.random_bf16((H, r), seed=80, std=0.01)
    L2d = inputs.random_bf16((r, D), seed=81, std=0.01)
    bd = inputs.random_bf16((D,), seed=82, std=0.01)
    X = dev_bf16(du["X"])
    Wq_u, ws_u = w4.w4a4_quantize_weights(dev_bf16(du["W"]), g)
    Wq_d, ws_d = w4.w4a4_quantize_weights(dev_bf16(Wd), g)
    up = dict(Wq=Wq_u, w_scale=ws_u, L1=dev_bf16(du["L1"]), L2=dev_bf16(du["L2"]), bias=dev_bf16(du["bias"]))
    down = dict(Wq=Wq_d, w_scale=ws_d, L1=dev_bf16(L1d), L2=dev_bf16(L2d), bias=dev_bf16(bd))
    Y = w4.w4a4_mlp(X, g, up, down)
    h = w4.w4a4_linear_gelu(X, Wq_u, ws_u, g, up["L1"], up["L2"], up["bias"])
    Y2 = w4.w4a4_linear(h, Wq_d, ws_d, g, down["L1"], down["L2"], down["bias"])
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    ref_h = oracle.linear_w4a4_gelu(du["X"], du["W"], g, du["L1"], du["L2"], du["bias"])
    check_output(host_f64(h), ref_h["Y"], lowrank=True)
    h_bits = h.cpu().view(torch.int16).numpy().view(np.uint16)
    ref_y = oracle.linear_w4a4(h_bits, Wd, g, L1d, L2d, bd)
    check_output(host_f64(Y), ref_y["Y"], lowrank=True)


@pytest.mark.parametrize("N,K,g,rl,scale,seed", [(264, 640, 64, 16, 0.5, 1), (96, 3072, 128, 64, 1.3, 77),
                                                 (40, 12288, 128, 32, 0.7, 2 ** 63 + 11), (64, 256, 0, 16, 2.0, 5)])
def test_bake_lora_sr_bitexact(N, K, g, rl, scale, seed):
    """LoRA baked into W (bf16, fp32 index-order FMA sums) and stochastically
    re-quantized with Philox4x64-10: the baked weights, scales and codes are
    bit-identical to the oracle's, and a second call with the same seed
    repeats them."""
    import torch
    W = inputs.random_bf16((N, K), seed=N + K, std=0.02)
    A = inputs.random_bf16((K, rl), seed=rl, std=0.05)
    B = inputs.random_bf16((rl, N), seed=rl + 1, std=0.05)
    Wb, Wq, ws = w4.w4a4_bake_lora_sr(dev_bf16(W), dev_bf16(A), dev_bf16(B), scale, g, seed)
    torch.cuda.synchronize()
    ref = oracle.bake_requantize(W, A, B, scale, g, seed)
    assert np.array_equal(Wb.cpu().view(torch.int16).numpy().view(np.uint16), ref["w_baked"])
    assert np.array_equal(ws.cpu().numpy().view(np.uint32), ref["w_scale"].view(np.uint32))
    got = Wq.cpu().numpy()
    assert np.array_equal(got, ref["w_packed"]), f"{np.count_nonzero(got != ref['w_packed'])} code bytes differ"
    _, Wq2, _ = w4.w4a4_bake_lora_sr(dev_bf16(W), dev_bf16(A), dev_bf16(B), scale, g, seed)
    assert torch.equal(Wq2, Wq)


def test_attn_proj_full_size_sampled():
    """The attention-projection workload at full size (M=4608, K=N=3072,
    g=128, bias), in the launch configuration the benchmark times
    (w4a4_linear), checked on sampled token rows the oracle computes one by
    one, plus bit-exact accumulators of those rows."""
    import torch
    spec = inputs.WORKLOADS["attn_proj"]
    d = inputs.make_layer(spec)
    X, W, b = dev_bf16(d["X"]), dev_bf16(d["W"]), dev_bf16(d["bias"])
    Wq, ws = w4.w4a4_quantize_weights(W, spec.group)
    Y = w4.w4a4_linear(X, Wq, ws, spec.group, bias=b)
    Xq, xs, _ = w4.w4a4_rotate_quantize_act(X, spec.group)
    acc = torch.empty((spec.M, spec.N), dtype=torch.int32, device="cuda")
    w4.w4a4_gemm(Xq, xs, Wq, ws, spec.group, bias=b, acc_debug=acc)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(5).choice(spec.M, size=40, replace=False))
    rows = np.unique(np.concatenate([rows, [0, spec.M - 1]]))
    wp, wsr, wq = oracle.quantize_w4(d["W"], spec.group)
    assert np.array_equal(Wq.cpu().numpy(), wp)
    assert np.array_equal(ws.cpu().numpy(), wsr)
    xp, xsr, xq = oracle.quantize_w4(d["X"][rows], spec.group)
    assert np.array_equal(Xq.cpu().numpy()[rows], xp)
    acc_ref = oracle.int_gemm(xq, wq)
    assert np.array_equal(acc.cpu().numpy()[rows], acc_ref)
    y_ref = oracle.epilogue(acc_ref, xsr, wsr, spec.group, None, None, d["bias"])
    check_output(host_f64(Y)[rows], y_ref, lowrank=False)


@pytest.mark.parametrize("name", ["mlp_up", "mlp_down"])
def test_mlp_layers_full_size_sampled(name):
    """The MLP layers at full size (M=4608, 3072->12288 and 12288->3072,
    g=128, r=128, bias) in the benchmark's launch configuration
    (w4a4_linear), on sampled token rows: weight and activation codes and
    scales, the low-rank T, bit-exact accumulators of those rows, outputs
    within the low-rank tolerance."""
    import torch
    spec = inputs.WORKLOADS[name]
    d = inputs.make_layer(spec)
    X, W, b = dev_bf16(d["X"]), dev_bf16(d["W"]), dev_bf16(d["bias"])
    L1, L2 = dev_bf16(d["L1"]), dev_bf16(d["L2"])
    Wq, ws = w4.w4a4_quantize_weights(W, spec.group)
    Y = w4.w4a4_linear(X, Wq, ws, spec.group, L1, L2, b)
    Xq, xs, T = w4.w4a4_rotate_quantize_act(X, spec.group, L1)
    acc = torch.empty((spec.M, spec.N), dtype=torch.int32, device="cuda")
    w4.w4a4_gemm(Xq, xs, Wq, ws, spec.group, T, L2, b, acc_debug=acc)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(6).choice(spec.M, size=24, replace=False))
    rows = np.unique(np.concatenate([rows, [0, spec.M - 1]]))
    wp, wsr, wq = oracle.quantize_w4(d["W"], spec.group)
    assert np.array_equal(Wq.cpu().numpy(), wp)
    assert np.array_equal(ws.cpu().numpy(), wsr)
    xp, xsr, xq = oracle.quantize_w4(d["X"][rows], spec.group)
    assert np.array_equal(Xq.cpu().numpy()[rows], xp)
    assert np.array_equal(xs.cpu().numpy()[rows], xsr)
    acc_ref = oracle.int_gemm(xq, wq)
    assert np.array_equal(acc.cpu().numpy()[rows], acc_ref)
    t_ref = oracle.lowrank_down(d["X"][rows], d["L1"])
    assert np.max(np.abs(host_f64(T)[rows] - t_ref)) <= 1e-2 * np.max(np.abs(t_ref))
    y_ref = oracle.epilogue(acc_ref, xsr, wsr, spec.group, t_ref, d["L2"], d["bias"])
    check_output(host_f64(Y)[rows], y_ref, lowrank=True)


def test_block_layers_full_size_sampled():
    """The double-stream block at batch 2 (M=9216): the fused QKV projection
    (3072 -> 9216, r=64) through w4a4_linear and the W8A8 first projection
    (3072 -> 3072) through w8a8_linear, on sampled token rows: codes, scales
    and accumulators bit-exact, outputs within tolerance."""
    import torch
    spec = inputs.WORKLOADS["block_qkv"]
    d = inputs.make_layer(spec)
    X, W, L1, L2 = dev_bf16(d["X"]), dev_bf16(d["W"]), dev_bf16(d["L1"]), dev_bf16(d["L2"])
    b = dev_bf16(d["bias"]) if d["bias"] is not None else None
    Wq, ws = w4.w4a4_quantize_weights(W, spec.group)
    Y = w4.w4a4_linear(X, Wq, ws, spec.group, L1, L2, b)
    Xq, xs, T = w4.w4a4_rotate_quantize_act(X, spec.group, L1)
    acc = torch.empty((spec.M, spec.N), dtype=torch.int32, device="cuda")
    w4.w4a4_gemm(Xq, xs, Wq, ws, spec.group, T, L2, b, acc_debug=acc)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.random.default_rng(7).choice(spec.M, size=16, replace=False),
                                     [0, spec.M - 1]]))
    wp, wsr, wq = oracle.quantize_w4(d["W"], spec.group)
    assert np.array_equal(Wq.cpu().numpy(), wp) and np.array_equal(ws.cpu().numpy(), wsr)
    xp, xsr, xq = oracle.quantize_w4(d["X"][rows], spec.group)
    assert np.array_equal(Xq.cpu().numpy()[rows], xp)
    acc_ref = oracle.int_gemm(xq, wq)
    assert np.array_equal(acc.cpu().numpy()[rows], acc_ref)
    t_ref = oracle.lowrank_down(d["X"][rows], d["L1"])
    y_ref = oracle.epilogue(acc_ref, xsr, wsr, spec.group, t_ref, d["L2"], d["bias"])
    check_output(host_f64(Y)[rows], y_ref, lowrank=True)

    spec8 = inputs.WORKLOADS["block_first_w8a8"]
    d8 = inputs.make_layer(spec8)
    X8, W8 = dev_bf16(d8["X"]), dev_bf16(d8["W"])
    b8 = dev_bf16(d8["bias"]) if d8["bias"] is not None else None
    Wq8, ws8 = w4.w8a8_quantize_weights(W8, spec8.group)
    Y8 = w4.w8a8_linear(X8, Wq8, ws8, spec8.group, b8)
    torch.cuda.synchronize()
    wq8, wsr8 = oracle.quantize_w8(d8["W"], spec8.group)
    assert np.array_equal(Wq8.cpu().numpy(), wq8) and np.array_equal(ws8.cpu().numpy(), wsr8)
    xq8, xsr8 = oracle.quantize_w8(d8["X"][rows], spec8.group)
    acc8 = oracle.int_gemm(xq8, wq8)
    y8_ref = oracle.epilogue(acc8, xsr8, wsr8, spec8.group, None, None, d8["bias"])
    check_output(host_f64(Y8)[rows], y8_ref, lowrank=False)


def test_no_device_error_after_runs():
    assert w4.w4a4_get_device_error() == 0
