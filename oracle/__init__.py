"""CPU oracle for the W4A4 ConvRot linear layer (and the W8A8 and W4A8 twins).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA path and never imports it.

Every step calls the plain C routines in ``oracle.c`` (explicit Hadamard
matrix, tree-order fp32 sums, IEEE fp32 quantization, int64 GEMM, fp64
epilogue); this module only marshals NumPy arrays.  bf16 tensors are passed
as ``uint16`` arrays holding the bf16 bit patterns.

Sources restated (the pages give prose, no formulas):
  * "Load Diffusion Model INT4 (W4A4)" (comfy.icu), intro: rotate with a
    Hadamard transform first, then quantize to 4 bit, then integer matmul.
  * "W4A4 and W4A8: The New Quantization Toolkit" (renderbob.io), "Decoding the
    notation": weights quantized once, activations on the fly.
  * "Krea 2 Turbo - SVDQuant" (sweettea.co), "Why activation-aware INT4",
    "What's included": Hadamard step for outliers, parallel low-rank branch.
  * "ComfyUI-INT4-Fast" (kongchang.com), "Per-Layer Dynamic Routing": the INT8
    path for sensitive layers.

Pins: tests/test_oracle_pins.py checks each function against facts that do
not come from this code (H H^T = gI and scipy's Sylvester Hadamard, the fp64
rotation identity, an independently coded fp32 FWHT, the quantization error
bound, closed-form rows, a NumPy int64 matmul, hand-derived golden fixtures).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        L = ctypes.c_long
        I = ctypes.c_int
        lib.oracle_num_threads.restype = I
        lib.oracle_hadamard.argtypes = [I, P]
        lib.oracle_rotate.argtypes = [P, L, I, I, P]
        lib.oracle_rotate.restype = I
        lib.oracle_quantize.argtypes = [P, L, I, I, P, P]
        lib.oracle_quantize_asym4.argtypes = [P, L, I, P, P, P]
        lib.oracle_pack_int4.argtypes = [P, L, I, P]
        lib.oracle_unpack_int4.argtypes = [P, L, I, P]
        lib.oracle_int_gemm.argtypes = [P, P, L, L, I, P]
        lib.oracle_int_gemm.restype = L
        lib.oracle_lowrank_down.argtypes = [P, P, L, I, I, P]
        lib.oracle_epilogue.argtypes = [P, P, P, L, L, I, P, P, I, P, P]
        lib.oracle_f32_to_bf16.argtypes = [P, L, P]
        lib.oracle_f64_to_bf16.argtypes = [P, L, P]
        lib.oracle_lora_merge.argtypes = [P, P, I, P, P, I, ctypes.c_float, I, I, P, P]
        lib.oracle_lowrank_up.argtypes = [P, P, L, L, I, ctypes.c_double, P]
        lib.oracle_gelu_tanh.argtypes = [P, L, P]
        lib.oracle_philox4x64.argtypes = [P, P, P]
        lib.oracle_sr_uniform.argtypes = [L, ctypes.c_uint64, P]
        lib.oracle_lora_bake.argtypes = [P, P, P, I, I, I, ctypes.c_float, P]
        lib.oracle_quantize_sr.argtypes = [P, L, I, P, P, P]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _bf16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 tensors are passed as uint16 bit patterns")
    return a


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def hadamard(g: int) -> np.ndarray:
    """Sylvester Hadamard matrix H_g[i][j] = (-1)^popcount(i & j), int8."""
    H = np.empty((g, g), dtype=np.int8)
    _load().oracle_hadamard(g, _ptr(H))
    return H


def rotate(X: np.ndarray, g: int) -> np.ndarray:
    """Block-diagonal Hadamard rotation of each bf16 row, fp32 tree-order sums."""
    X = _bf16(X)
    rows, K = X.shape
    Y = np.empty((rows, K), dtype=np.float32)
    rc = _load().oracle_rotate(_ptr(X), rows, K, g, _ptr(Y))
    if rc != 0:
        raise ValueError(f"rotate: group {g} does not divide K={K} or is not a power of two")
    return Y


def quantize(Y: np.ndarray, qmax: int) -> tuple[np.ndarray, np.ndarray]:
    """Per-row symmetric absmax quantization in IEEE fp32 -> (int8 codes, fp32 scales)."""
    Y = np.ascontiguousarray(Y, dtype=np.float32)
    rows, K = Y.shape
    q = np.empty((rows, K), dtype=np.int8)
    s = np.empty((rows,), dtype=np.float32)
    _load().oracle_quantize(_ptr(Y), rows, K, qmax, _ptr(q), _ptr(s))
    return q, s


def quantize_asym4(Y: np.ndarray) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Per-row asymmetric 4-bit quantization with a zero point in IEEE fp32
    -> (uint8 codes 0..15, fp32 scales, uint8 zero points)."""
    Y = np.ascontiguousarray(Y, dtype=np.float32)
    rows, K = Y.shape
    q = np.empty((rows, K), dtype=np.uint8)
    s = np.empty((rows,), dtype=np.float32)
    z = np.empty((rows,), dtype=np.uint8)
    _load().oracle_quantize_asym4(_ptr(Y), rows, K, _ptr(q), _ptr(s), _ptr(z))
    return q, s, z


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Two codes per byte, even k in the low nibble (4-bit two's complement for
    signed codes; the same bits for unsigned codes 0..15)."""
    q = np.ascontiguousarray(q).astype(np.int8)
    rows, K = q.shape
    out = np.empty((rows, K // 2), dtype=np.uint8)
    _load().oracle_pack_int4(_ptr(q), rows, K, _ptr(out))
    return out


def unpack_int4(p: np.ndarray, K: int) -> np.ndarray:
    p = np.ascontiguousarray(p, dtype=np.uint8)
    rows = p.shape[0]
    q = np.empty((rows, K), dtype=np.int8)
    _load().oracle_unpack_int4(_ptr(p), rows, K, _ptr(q))
    return q


def int_gemm(qa: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """acc = qa @ qw.T exactly (int64 sums stored as int32; raises on overflow)."""
    qa = np.ascontiguousarray(qa, dtype=np.int8)
    qw = np.ascontiguousarray(qw, dtype=np.int8)
    M, K = qa.shape
    N, K2 = qw.shape
    assert K == K2
    acc = np.empty((M, N), dtype=np.int32)
    ov = _load().oracle_int_gemm(_ptr(qa), _ptr(qw), M, N, K, _ptr(acc))
    if ov:
        raise OverflowError(f"{ov} accumulators exceed int32")
    return acc


def lowrank_down(X: np.ndarray, L1: np.ndarray) -> np.ndarray:
    """T = X @ L1 in fp64 from bf16 X [M,K] and bf16 L1 [K,r]."""
    X = _bf16(X)
    L1 = _bf16(L1)
    M, K = X.shape
    K2, r = L1.shape
    assert K == K2
    T = np.empty((M, r), dtype=np.float64)
    _load().oracle_lowrank_down(_ptr(X), _ptr(L1), M, K, r, _ptr(T))
    return T


def epilogue(acc, sa, sw, g, T=None, L2=None, bias=None) -> np.ndarray:
    """Y = acc*sa*sw/g + T@L2 + bias in fp64 (unrounded)."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, N = acc.shape
    r = 0
    if T is not None:
        T = np.ascontiguousarray(T, dtype=np.float64)
        L2 = _bf16(L2)
        r = T.shape[1]
        assert L2.shape == (r, N)
    if bias is not None:
        bias = _bf16(bias)
        assert bias.shape == (N,)
    Y = np.empty((M, N), dtype=np.float64)
    _load().oracle_epilogue(_ptr(acc), _ptr(sa), _ptr(sw), M, N, g,
                            _ptr(T) if r else None, _ptr(L2) if r else None, r,
                            _ptr(bias), _ptr(Y))
    return Y


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_f32_to_bf16(_ptr(x), x.size, _ptr(out))
    return out


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_f64_to_bf16(_ptr(x), x.size, _ptr(out))
    return out


def bf16_to_f64(h: np.ndarray) -> np.ndarray:
    h = _bf16(h)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---- composed steps of the layer -------------------------------------------------

def quantize_w4(X: np.ndarray, g: int):
    """Rotate + per-row INT4 quantize + pack.  Same routine for activations
    (one scale per token) and weights (one scale per output channel)."""
    q, s = quantize(rotate(X, g), 7)
    return pack_int4(q), s, q


def quantize_w8(X: np.ndarray, g: int):
    """Rotate + per-row symmetric INT8 quantize (W8A8 fallback)."""
    q, s = quantize(rotate(X, g), 127)
    return q, s


def linear_w4a4(X, W, g, L1=None, L2=None, bias=None):
    """Full W4A4 ConvRot layer on bf16 inputs -> dict of every intermediate."""
    xp, xs, xq = quantize_w4(X, g)
    wp, ws, wq = quantize_w4(W, g)
    acc = int_gemm(xq, wq)
    T = lowrank_down(X, L1) if L1 is not None else None
    Y = epilogue(acc, xs, ws, g, T, L2 if T is not None else None, bias)
    return dict(x_packed=xp, x_scale=xs, x_q=xq, w_packed=wp, w_scale=ws, w_q=wq,
                acc=acc, T=T, Y=Y)


def quantize_w4a8_weights(W: np.ndarray, g: int):
    """Rotate + per-output-channel asymmetric 4-bit quantize + pack (W4A8)."""
    q, s, z = quantize_asym4(rotate(W, g))
    return pack_int4(q), s, z, q


def linear_w4a8(X, W, g, bias=None):
    """W4A8 layer: rotated per-token INT8 activations (as in W8A8) times
    rotated asymmetric 4-bit weights; acc = sum_k qa * (qw - z) exactly."""
    xq, xs = quantize_w8(X, g)
    wp, ws, wz, wq = quantize_w4a8_weights(W, g)
    centered = (wq.astype(np.int16) - wz.astype(np.int16)[:, None]).astype(np.int8)
    acc = int_gemm(xq, centered)
    Y = epilogue(acc, xs, ws, g, None, None, bias)
    return dict(x_q=xq, x_scale=xs, w_packed=wp, w_scale=ws, w_zero=wz, w_q=wq, acc=acc, Y=Y)


def philox4x64(counter, key) -> np.ndarray:
    """Philox4x64-10 block for a 4-word counter and 2-word key (uint64)."""
    c = np.ascontiguousarray(counter, dtype=np.uint64)
    k = np.ascontiguousarray(key, dtype=np.uint64)
    out = np.empty(4, dtype=np.uint64)
    _load().oracle_philox4x64(_ptr(c), _ptr(k), _ptr(out))
    return out


def sr_uniform(n: int, seed: int) -> np.ndarray:
    """The u in [0, 1) of elements 0..n-1 of a row-major array (fp32)."""
    u = np.empty(n, dtype=np.float32)
    _load().oracle_sr_uniform(n, seed, _ptr(u))
    return u


def lora_bake(W, A, B, scale: float) -> np.ndarray:
    """bf16(W + scale * (A @ B)^T), fp32 index-order FMA sums."""
    W, A, B = _bf16(W), _bf16(A), _bf16(B)
    N, K = W.shape
    rl = A.shape[1]
    Wb = np.empty((N, K), dtype=np.uint16)
    _load().oracle_lora_bake(_ptr(W), _ptr(A), _ptr(B), N, K, rl, float(scale), _ptr(Wb))
    return Wb


def quantize_sr(Y: np.ndarray, U: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Per-row absmax INT4 scale, stochastic rounding with the given u."""
    Y = np.ascontiguousarray(Y, dtype=np.float32)
    U = np.ascontiguousarray(U, dtype=np.float32).reshape(Y.shape)
    rows, K = Y.shape
    q = np.empty((rows, K), dtype=np.int8)
    s = np.empty((rows,), dtype=np.float32)
    _load().oracle_quantize_sr(_ptr(Y), rows, K, _ptr(U), _ptr(q), _ptr(s))
    return q, s


def bake_requantize(W, A, B, scale: float, g: int, seed: int):
    """LoRA baked into W, then rotated and stochastically rounded to INT4."""
    Wb = lora_bake(W, A, B, scale)
    Y = rotate(Wb, g)
    q, s = quantize_sr(Y, sr_uniform(Y.size, seed).reshape(Y.shape))
    return dict(w_baked=Wb, w_q=q, w_scale=s, w_packed=pack_int4(q))


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """GELU, tanh approximation, in fp64."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    _load().oracle_gelu_tanh(_ptr(x), x.size, _ptr(y))
    return y


def linear_w4a4_gelu(X, W, g, L1=None, L2=None, bias=None):
    """W4A4 layer followed by GELU(tanh) on its unrounded output (fp64): the
    fused up-projection of the MLP."""
    out = linear_w4a4(X, W, g, L1, L2, bias)
    out = dict(out)
    out["Y_linear"] = out["Y"]
    out["Y"] = gelu_tanh(out["Y"])
    return out


def lora_merge(L1, L2, A, B, scale: float):
    """Low-rank operands of the merged branch: ([L1 | A], [L2 ; bf16(scale * B)])."""
    A = _bf16(A)
    B = _bf16(B)
    K, rl = A.shape
    N = B.shape[1]
    r = 0 if L1 is None else L1.shape[1]
    L1 = _bf16(L1) if r else np.zeros((K, 0), np.uint16)
    L2 = _bf16(L2) if r else np.zeros((0, N), np.uint16)
    L1o = np.empty((K, r + rl), dtype=np.uint16)
    L2o = np.empty((r + rl, N), dtype=np.uint16)
    _load().oracle_lora_merge(_ptr(L1) if r else None, _ptr(L2) if r else None, r, _ptr(A), _ptr(B), rl,
                              float(scale), K, N, _ptr(L1o), _ptr(L2o))
    return L1o, L2o


def linear_w4a4_lora(X, W, g, L1, L2, A, B, scale: float, bias=None):
    """W4A4 layer with the SVDQuant branch and a runtime LoRA beside it:
    Y = dequant(acc) + (X L1) L2 + scale (X A) B + bias, the low-rank terms in
    fp64 from the bf16 operands (unmerged)."""
    base = linear_w4a4(X, W, g, L1, L2, bias)
    TA = lowrank_down(X, A)
    out = dict(base)
    out["Y"] = lowrank_up(TA, B, float(np.float32(scale)), base["Y"])
    out["T_lora"] = TA
    return out


def lowrank_up(T, U, scale: float, Y):
    """Y + scale * (T U) in fp64 (oracle_lowrank_up): T fp64 [M, r], U bf16
    bits [r, N], Y fp64 [M, N]; returns a new array."""
    T = np.ascontiguousarray(T, dtype=np.float64)
    U = _bf16(U)
    M, r = T.shape
    N = U.shape[1]
    out = np.array(Y, dtype=np.float64, order="C", copy=True)
    _load().oracle_lowrank_up(_ptr(T), _ptr(U), M, N, r, float(scale), _ptr(out))
    return out


def linear_w8a8(X, W, g, bias=None):
    xq, xs = quantize_w8(X, g)
    wq, ws = quantize_w8(W, g)
    acc = int_gemm(xq, wq)
    Y = epilogue(acc, xs, ws, g, None, None, bias)
    return dict(x_q=xq, x_scale=xs, w_q=wq, w_scale=ws, acc=acc, Y=Y)
