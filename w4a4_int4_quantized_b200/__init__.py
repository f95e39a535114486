"""Python binding of libw4a4 (the W4A4 ConvRot INT4 linear layer for B200).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libw4a4.so`` behind the C ABI declared in ``include/w4a4.h``.  PyTorch
provides device memory and the stream (``torch.cuda.current_stream()`` unless
one is given).  Functions carry the C names; outputs not passed in are
allocated with torch before the call.  There is no CPU fallback: if the
library is missing or a call fails, a ``W4A4Error`` is raised.

bf16 tensors are torch.bfloat16; packed INT4 codes are torch.uint8 [rows, K/2];
INT8 codes are torch.int8 [rows, K]; scales are torch.float32 [rows].
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "W4A4Error", "library_path", "load_library",
    "w4a4_version", "w4a4_status_string",
    "w4a4_quantize_weights", "w4a4_rotate_quantize_act", "w4a4_gemm", "w4a4_linear",
    "w4a4_workspace_bytes", "w4a4_linear_noalloc", "NOALLOC_SCRATCH_BYTES",
    "w8a8_quantize_weights", "w8a8_rotate_quantize_act", "w8a8_gemm", "w8a8_linear",
    "w8a8_workspace_bytes", "w4a8_quantize_weights", "w4a8_gemm", "w4a8_linear", "w4a8_workspace_bytes",
    "w4a4_lora_merge", "w4a4_gemm_gelu", "w4a4_linear_gelu", "w4a4_mlp", "w4a4_mlp_workspace_bytes",
    "w4a4_bake_lora_sr", "w4a4_get_device_error", "w4a4_selftest_wait_timeout", "w4a4_plan_rotate_quantize",
    "w4a4_plan_gemm_split",
    "DEVERR_WAIT_OPERANDS", "DEVERR_WAIT_SLOT", "DEVERR_WAIT_ACCUM", "DEVERR_WAIT_DRAIN",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libw4a4.so")
_lib = None

W4A4_OK = 0
# bits of the device error word (W4A4_DEVERR_* in include/w4a4.h)
DEVERR_WAIT_OPERANDS, DEVERR_WAIT_SLOT, DEVERR_WAIT_ACCUM, DEVERR_WAIT_DRAIN = 1, 2, 4, 8
STATUS = {
    0: "W4A4_OK", 1: "W4A4_ERR_INVALID_ARG", 2: "W4A4_ERR_UNSUPPORTED_SHAPE", 3: "W4A4_ERR_MISALIGNED",
    4: "W4A4_ERR_CUDA", 5: "W4A4_ERR_DEVICE_TIMEOUT", 6: "W4A4_ERR_UNSUPPORTED_DEVICE", 7: "W4A4_ERR_WORKSPACE",
}


class W4A4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libw4a4.so and declare the C signatures (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise W4A4Error("load_library", 4) from FileNotFoundError(
            f"{_LIB_PATH} not built; run __graft_entry__.build() or python -m w4a4_int4_quantized_b200.build")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, Z, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_int
    sig = {
        "w4a4_version": ([], I),
        "w4a4_status_string": ([I], ctypes.c_char_p),
        "w4a4_quantize_weights": ([P, I, I, I, P, P, P], S),
        "w4a4_rotate_quantize_act": ([P, I, I, I, P, P, P, I, P, P], S),
        "w4a4_gemm": ([P, P, P, P, I, I, I, I, P, P, I, P, P, P, P], S),
        "w4a4_workspace_bytes": ([I, I, I], Z),
        "w4a4_linear": ([P, P, P, I, I, I, I, P, P, I, P, P, P, Z, P], S),
        "w4a4_linear_noalloc": ([P, P, P, I, I, I, I, P, P, I, P, P, P], S),
        "w8a8_quantize_weights": ([P, I, I, I, P, P, P], S),
        "w8a8_rotate_quantize_act": ([P, I, I, I, P, P, P], S),
        "w8a8_gemm": ([P, P, P, P, I, I, I, I, P, P, P, P], S),
        "w8a8_workspace_bytes": ([I, I], Z),
        "w8a8_linear": ([P, P, P, I, I, I, I, P, P, P, Z, P], S),
        "w4a8_quantize_weights": ([P, I, I, I, P, P, P, P], S),
        "w4a8_gemm": ([P, P, P, P, P, I, I, I, I, P, P, P, P], S),
        "w4a8_workspace_bytes": ([I, I], Z),
        "w4a8_linear": ([P, P, P, P, I, I, I, I, P, P, P, Z, P], S),
        "w4a4_lora_merge": ([P, P, I, P, P, I, ctypes.c_float, I, I, P, P, P], S),
        "w4a4_gemm_gelu": ([P, P, P, P, I, I, I, I, P, P, I, P, P, P, P], S),
        "w4a4_linear_gelu": ([P, P, P, I, I, I, I, P, P, I, P, P, P, Z, P], S),
        "w4a4_mlp_workspace_bytes": ([I, I, I, I, I], Z),
        "w4a4_bake_lora_sr": ([P, P, P, I, ctypes.c_float, I, I, I, ctypes.c_ulonglong, P, P, P, P], S),
        "w4a4_mlp": ([P, I, I, I, I, P, P, P, P, I, P, P, P, P, P, I, P, P, P, Z, P], S),
        "w4a4_get_device_error": ([P, ctypes.POINTER(ctypes.c_uint)], S),
        "w4a4_selftest_wait_timeout": ([P, P, I, I, I, P, ctypes.c_uint, P], S),
        "w4a4_plan_rotate_quantize": ([I, I, I, I, I, I, ctypes.POINTER(ctypes.c_int)], S),
        "w4a4_plan_gemm_split": ([I, I, I, I, I, I, I, ctypes.POINTER(ctypes.c_int)], S),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, status: int):
    if status != W4A4_OK:
        raise W4A4Error(fn, status)


def _empty(shape, dtype, like):
    import torch
    return torch.empty(shape, dtype=dtype, device=like.device)


def w4a4_version() -> int:
    return load_library().w4a4_version()


def w4a4_status_string(status: int) -> str:
    return load_library().w4a4_status_string(status).decode()


def w4a4_quantize_weights(W, group, Wq=None, w_scale=None, stream=None):
    import torch
    N, K = W.shape
    Wq = _empty((N, K // 2), torch.uint8, W) if Wq is None else Wq
    w_scale = _empty((N,), torch.float32, W) if w_scale is None else w_scale
    _check("w4a4_quantize_weights", load_library().w4a4_quantize_weights(
        _ptr(W), N, K, group, _ptr(Wq), _ptr(w_scale), _stream(stream)))
    return Wq, w_scale


def w4a4_rotate_quantize_act(X, group, L1=None, Xq=None, x_scale=None, T=None, stream=None):
    import torch
    M, K = X.shape
    rank = 0 if L1 is None else L1.shape[1]
    Xq = _empty((M, K // 2), torch.uint8, X) if Xq is None else Xq
    x_scale = _empty((M,), torch.float32, X) if x_scale is None else x_scale
    if rank and T is None:
        T = _empty((M, rank), torch.bfloat16, X)
    _check("w4a4_rotate_quantize_act", load_library().w4a4_rotate_quantize_act(
        _ptr(X), M, K, group, _ptr(Xq), _ptr(x_scale), _ptr(L1), rank, _ptr(T) if rank else None,
        _stream(stream)))
    return Xq, x_scale, (T if rank else None)


def w4a4_gemm(Xq, x_scale, Wq, w_scale, group, T=None, L2=None, bias=None, Y=None, acc_debug=None,
              stream=None):
    import torch
    M = Xq.shape[0]
    N = Wq.shape[0]
    K = Xq.shape[1] * 2
    rank = 0 if L2 is None else L2.shape[0]
    Y = _empty((M, N), torch.bfloat16, Xq) if Y is None else Y
    _check("w4a4_gemm", load_library().w4a4_gemm(
        _ptr(Xq), _ptr(x_scale), _ptr(Wq), _ptr(w_scale), M, N, K, group, _ptr(T), _ptr(L2), rank,
        _ptr(bias), _ptr(Y), _ptr(acc_debug), _stream(stream)))
    return Y


def w4a4_workspace_bytes(M: int, K: int, rank: int) -> int:
    return int(load_library().w4a4_workspace_bytes(M, K, rank))


def w4a4_linear(X, Wq, w_scale, group, L1=None, L2=None, bias=None, Y=None, workspace=None, stream=None):
    import torch
    M, K = X.shape
    N = Wq.shape[0]
    rank = 0 if L1 is None else L1.shape[1]
    need = w4a4_workspace_bytes(M, K, rank)
    if workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=X.device)
    Y = _empty((M, N), torch.bfloat16, X) if Y is None else Y
    _check("w4a4_linear", load_library().w4a4_linear(
        _ptr(X), _ptr(Wq), _ptr(w_scale), M, N, K, group, _ptr(L1), _ptr(L2), rank, _ptr(bias), _ptr(Y),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return Y


NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024   # W4A4_NOALLOC_SCRATCH_BYTES in include/w4a4.h


def w4a4_linear_noalloc(X, Wq, w_scale, group, L1=None, L2=None, bias=None, Y=None, stream=None):
    """w4a4_linear on the library's built-in scratch: the C call allocates no
    device memory (Y is allocated here with torch only when not passed in).
    Layers needing more than NOALLOC_SCRATCH_BYTES of scratch are rejected."""
    import torch
    M, K = X.shape
    N = Wq.shape[0]
    rank = 0 if L1 is None else L1.shape[1]
    Y = _empty((M, N), torch.bfloat16, X) if Y is None else Y
    _check("w4a4_linear_noalloc", load_library().w4a4_linear_noalloc(
        _ptr(X), _ptr(Wq), _ptr(w_scale), M, N, K, group, _ptr(L1), _ptr(L2), rank, _ptr(bias), _ptr(Y),
        _stream(stream)))
    return Y


def w8a8_quantize_weights(W, group, Wq=None, w_scale=None, stream=None):
    import torch
    N, K = W.shape
    Wq = _empty((N, K), torch.int8, W) if Wq is None else Wq
    w_scale = _empty((N,), torch.float32, W) if w_scale is None else w_scale
    _check("w8a8_quantize_weights", load_library().w8a8_quantize_weights(
        _ptr(W), N, K, group, _ptr(Wq), _ptr(w_scale), _stream(stream)))
    return Wq, w_scale


def w8a8_rotate_quantize_act(X, group, Xq=None, x_scale=None, stream=None):
    import torch
    M, K = X.shape
    Xq = _empty((M, K), torch.int8, X) if Xq is None else Xq
    x_scale = _empty((M,), torch.float32, X) if x_scale is None else x_scale
    _check("w8a8_rotate_quantize_act", load_library().w8a8_rotate_quantize_act(
        _ptr(X), M, K, group, _ptr(Xq), _ptr(x_scale), _stream(stream)))
    return Xq, x_scale


def w8a8_gemm(Xq, x_scale, Wq, w_scale, group, bias=None, Y=None, acc_debug=None, stream=None):
    import torch
    M, K = Xq.shape
    N = Wq.shape[0]
    Y = _empty((M, N), torch.bfloat16, Xq) if Y is None else Y
    _check("w8a8_gemm", load_library().w8a8_gemm(
        _ptr(Xq), _ptr(x_scale), _ptr(Wq), _ptr(w_scale), M, N, K, group, _ptr(bias), _ptr(Y),
        _ptr(acc_debug), _stream(stream)))
    return Y


def w8a8_workspace_bytes(M: int, K: int) -> int:
    return int(load_library().w8a8_workspace_bytes(M, K))


def w8a8_linear(X, Wq, w_scale, group, bias=None, Y=None, workspace=None, stream=None):
    import torch
    M, K = X.shape
    N = Wq.shape[0]
    need = w8a8_workspace_bytes(M, K)
    if workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=X.device)
    Y = _empty((M, N), torch.bfloat16, X) if Y is None else Y
    _check("w8a8_linear", load_library().w8a8_linear(
        _ptr(X), _ptr(Wq), _ptr(w_scale), M, N, K, group, _ptr(bias), _ptr(Y), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return Y


def w4a8_quantize_weights(W, group, Wq=None, w_scale=None, w_zero=None, stream=None):
    """Rotate + per-channel asymmetric 4-bit quantize: (packed codes [N, K/2],
    fp32 scales [N], uint8 zero points [N])."""
    import torch
    N, K = W.shape
    Wq = _empty((N, K // 2), torch.uint8, W) if Wq is None else Wq
    w_scale = _empty((N,), torch.float32, W) if w_scale is None else w_scale
    w_zero = _empty((N,), torch.uint8, W) if w_zero is None else w_zero
    _check("w4a8_quantize_weights", load_library().w4a8_quantize_weights(
        _ptr(W), N, K, group, _ptr(Wq), _ptr(w_scale), _ptr(w_zero), _stream(stream)))
    return Wq, w_scale, w_zero


def w4a8_gemm(Xq, x_scale, Wq, w_scale, w_zero, group, bias=None, Y=None, acc_debug=None, stream=None):
    import torch
    M, K = Xq.shape
    N = Wq.shape[0]
    Y = _empty((M, N), torch.bfloat16, Xq) if Y is None else Y
    _check("w4a8_gemm", load_library().w4a8_gemm(
        _ptr(Xq), _ptr(x_scale), _ptr(Wq), _ptr(w_scale), _ptr(w_zero), M, N, K, group, _ptr(bias), _ptr(Y),
        _ptr(acc_debug), _stream(stream)))
    return Y


def w4a8_workspace_bytes(M: int, K: int) -> int:
    return int(load_library().w4a8_workspace_bytes(M, K))


def w4a8_linear(X, Wq, w_scale, w_zero, group, bias=None, Y=None, workspace=None, stream=None):
    import torch
    M, K = X.shape
    N = Wq.shape[0]
    need = w4a8_workspace_bytes(M, K)
    if workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=X.device)
    Y = _empty((M, N), torch.bfloat16, X) if Y is None else Y
    _check("w4a8_linear", load_library().w4a8_linear(
        _ptr(X), _ptr(Wq), _ptr(w_scale), _ptr(w_zero), M, N, K, group, _ptr(bias), _ptr(Y), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return Y


def w4a4_lora_merge(L1, L2, A, B, lora_scale: float, L1_out=None, L2_out=None, stream=None):
    """Operands of the combined low-rank branch: ([L1 | A], [L2 ; bf16(scale B)]).
    L1 / L2 may be None (no SVDQuant branch)."""
    import torch
    K, rl = A.shape
    N = B.shape[1]
    r = 0 if L1 is None else L1.shape[1]
    L1_out = _empty((K, r + rl), torch.bfloat16, A) if L1_out is None else L1_out
    L2_out = _empty((r + rl, N), torch.bfloat16, A) if L2_out is None else L2_out
    _check("w4a4_lora_merge", load_library().w4a4_lora_merge(
        _ptr(L1), _ptr(L2), r, _ptr(A), _ptr(B), rl, float(lora_scale), K, N, _ptr(L1_out), _ptr(L2_out),
        _stream(stream)))
    return L1_out, L2_out


def w4a4_gemm_gelu(Xq, x_scale, Wq, w_scale, group, T=None, L2=None, bias=None, Y=None, acc_debug=None,
                   stream=None):
    """w4a4_gemm with GELU (tanh approximation) fused into the epilogue."""
    import torch
    M = Xq.shape[0]
    N, Kh = Wq.shape
    K = 2 * Kh
    rank = 0 if T is None else T.shape[1]
    Y = _empty((M, N), torch.bfloat16, Xq) if Y is None else Y
    _check("w4a4_gemm_gelu", load_library().w4a4_gemm_gelu(
        _ptr(Xq), _ptr(x_scale), _ptr(Wq), _ptr(w_scale), M, N, K, group, _ptr(T), _ptr(L2), rank, _ptr(bias),
        _ptr(Y), _ptr(acc_debug), _stream(stream)))
    return Y


def w4a4_linear_gelu(X, Wq, w_scale, group, L1=None, L2=None, bias=None, Y=None, workspace=None, stream=None):
    """w4a4_linear with GELU (tanh approximation) fused into the epilogue."""
    import torch
    M, K = X.shape
    N = Wq.shape[0]
    rank = 0 if L1 is None else L1.shape[1]
    need = w4a4_workspace_bytes(M, K, rank)
    if workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=X.device)
    Y = _empty((M, N), torch.bfloat16, X) if Y is None else Y
    _check("w4a4_linear_gelu", load_library().w4a4_linear_gelu(
        _ptr(X), _ptr(Wq), _ptr(w_scale), M, N, K, group, _ptr(L1), _ptr(L2), rank, _ptr(bias), _ptr(Y),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return Y


def w4a4_mlp_workspace_bytes(M: int, D: int, H: int, rank_up: int, rank_down: int) -> int:
    return int(load_library().w4a4_mlp_workspace_bytes(M, D, H, rank_up, rank_down))


def w4a4_mlp(X, group, up, down, Y=None, workspace=None, stream=None):
    """Y = down(gelu(up(X))).  up / down: dicts with Wq, w_scale and optional
    L1, L2, bias (the two layers' quantized weights and low-rank operands)."""
    import torch
    M, D = X.shape
    H = up["Wq"].shape[0]
    ru = 0 if up.get("L1") is None else up["L1"].shape[1]
    rd = 0 if down.get("L1") is None else down["L1"].shape[1]
    need = w4a4_mlp_workspace_bytes(M, D, H, ru, rd)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    Y = _empty((M, D), torch.bfloat16, X) if Y is None else Y
    _check("w4a4_mlp", load_library().w4a4_mlp(
        _ptr(X), M, D, H, group, _ptr(up["Wq"]), _ptr(up["w_scale"]), _ptr(up.get("L1")), _ptr(up.get("L2")), ru,
        _ptr(up.get("bias")), _ptr(down["Wq"]), _ptr(down["w_scale"]), _ptr(down.get("L1")),
        _ptr(down.get("L2")), rd, _ptr(down.get("bias")), _ptr(Y), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return Y


def w4a4_bake_lora_sr(W, A, B, lora_scale: float, group: int, seed: int, W_baked=None, Wq=None, w_scale=None,
                      stream=None):
    """LoRA baked into W, then rotated and stochastically rounded to INT4:
    (W_baked bf16 [N, K], packed codes [N, K/2], scales [N])."""
    import torch
    N, K = W.shape
    rl = A.shape[1]
    W_baked = _empty((N, K), torch.bfloat16, W) if W_baked is None else W_baked
    Wq = _empty((N, K // 2), torch.uint8, W) if Wq is None else Wq
    w_scale = _empty((N,), torch.float32, W) if w_scale is None else w_scale
    _check("w4a4_bake_lora_sr", load_library().w4a4_bake_lora_sr(
        _ptr(W), _ptr(A), _ptr(B), rl, float(lora_scale), N, K, group, int(seed), _ptr(W_baked), _ptr(Wq),
        _ptr(w_scale), _stream(stream)))
    return W_baked, Wq, w_scale


def w4a4_get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    code = ctypes.c_uint(0)
    status = load_library().w4a4_get_device_error(_stream(stream), ctypes.byref(code))
    if status not in (0, 5):
        raise W4A4Error("w4a4_get_device_error", status)
    return int(code.value)


def w4a4_selftest_wait_timeout(X, L1, timeout_us=1000, T=None, stream=None):
    """Run the low-rank down-projection with its operand loads withheld and the
    operand wait limited to `timeout_us`: the wait runs out, the kernel ends
    normally and the device error word then holds DEVERR_WAIT_OPERANDS.
    Returns T (undefined contents)."""
    import torch
    M, K = X.shape
    rank = L1.shape[1]
    T = _empty((M, rank), torch.bfloat16, X) if T is None else T
    _check("w4a4_selftest_wait_timeout", load_library().w4a4_selftest_wait_timeout(
        _ptr(X), _ptr(L1), M, K, rank, _ptr(T), timeout_us, _stream(stream)))
    return T


def w4a4_plan_rotate_quantize(M, K, group, sms=148, resident_per_sm=4, cached=True):
    """Launch shape the rotate + quantize kernel would use (host only, no CUDA
    call): (rows per block, threads, dynamic shared memory, grid)."""
    out = (ctypes.c_int * 4)()
    _check("w4a4_plan_rotate_quantize", load_library().w4a4_plan_rotate_quantize(
        M, K, group, sms, resident_per_sm, 1 if cached else 0, out))
    return tuple(out)


def w4a4_plan_gemm_split(M, N, K, rank=0, sms=148, clusters_of_8=16, clusters_of_4=32):
    """K slices the GEMM would split a layer over (4 or 2; 1 = the persistent
    form), for a device with `sms` SMs on which the given numbers of 8- and
    4-CTA clusters fit at once (host only, no CUDA call)."""
    out = ctypes.c_int(0)
    _check("w4a4_plan_gemm_split", load_library().w4a4_plan_gemm_split(
        M, N, K, rank, sms, clusters_of_8, clusters_of_4, ctypes.byref(out)))
    return out.value
