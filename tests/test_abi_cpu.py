"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/w4a4.h declares, and rejects bad arguments with the
documented status before launching anything."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

import w4a4_int4_quantized_b200 as w4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a4.h")

OK, INVALID, SHAPE, MISALIGNED, CUDA, TIMEOUT, DEVICE, WORKSPACE = range(8)

# fake device addresses: validation fails before any of them is dereferenced
A = ctypes.c_void_p(0x10000)
B = ctypes.c_void_p(0x20000)
C = ctypes.c_void_p(0x30000)
D = ctypes.c_void_p(0x40000)
E = ctypes.c_void_p(0x50000)
ODD = ctypes.c_void_p(0x10008)
NUL = None


@pytest.fixture(scope="module")
def lib():
    from w4a4_int4_quantized_b200 import build
    build.build()
    return w4.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b((?:w4a4|w8a8|w4a8)_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_documented_entry_points():
    names = _declared_functions()
    for n in ["w4a4_quantize_weights", "w4a4_rotate_quantize_act", "w4a4_gemm", "w4a4_linear",
              "w8a8_quantize_weights", "w8a8_rotate_quantize_act", "w8a8_gemm", "w8a8_linear",
              "w4a4_workspace_bytes", "w8a8_workspace_bytes", "w4a4_status_string", "w4a4_version",
              "w4a4_get_device_error", "w4a8_quantize_weights", "w4a8_gemm", "w4a8_linear",
              "w4a8_workspace_bytes", "w4a4_lora_merge", "w4a4_gemm_gelu", "w4a4_linear_gelu", "w4a4_mlp",
              "w4a4_mlp_workspace_bytes", "w4a4_bake_lora_sr"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert lib.w4a4_version() >= 100
    for code, name in w4.STATUS.items():
        assert lib.w4a4_status_string(code).decode() == name
    assert lib.w4a4_status_string(99).decode() == "W4A4_ERR_UNKNOWN"


def test_quantize_weights_validation(lib):
    f = lib.w4a4_quantize_weights
    assert f(NUL, 64, 256, 64, B, C, NUL) == INVALID
    assert f(A, 64, 256, 64, NUL, C, NUL) == INVALID
    assert f(A, 0, 256, 64, B, C, NUL) == SHAPE           # no rows
    assert f(A, 64, 192, 64, B, C, NUL) == SHAPE          # K not a multiple of 128
    assert f(A, 64, 256, 32, B, C, NUL) == SHAPE          # unsupported group
    assert f(A, 64, 256, 96, B, C, NUL) == SHAPE
    assert f(A, 64, 65536, 128, B, C, NUL) == SHAPE       # K / 128 > 256
    assert f(A, 64, 32768, 64, B, C, NUL) == SHAPE        # K / 64 > 256
    assert f(ODD, 64, 256, 64, B, C, NUL) == MISALIGNED
    assert f(A, 64, 256, 64, ODD, C, NUL) == MISALIGNED
    assert lib.w8a8_quantize_weights(A, 64, 256, 48, B, C, NUL) == SHAPE


def test_rotate_quantize_act_validation(lib):
    f = lib.w4a4_rotate_quantize_act
    assert f(A, 8, 256, 64, B, NUL, NUL, 0, NUL, NUL) == INVALID
    assert f(A, 8, 256, 64, B, C, NUL, 16, NUL, NUL) == INVALID        # rank without L1/T
    assert f(A, 8, 256, 64, B, C, D, 16, NUL, NUL) == INVALID
    assert f(A, 8, 256, 64, B, C, D, 24, E, NUL) == SHAPE              # rank not a multiple of 16
    assert f(A, 8, 256, 64, B, C, D, 272, E, NUL) == SHAPE             # rank > 256
    assert f(A, 8, 256, 64, B, C, ODD, 16, E, NUL) == MISALIGNED
    assert f(A, 0, 256, 64, B, C, NUL, 0, NUL, NUL) == SHAPE
    assert lib.w8a8_rotate_quantize_act(A, 8, 100, 0, B, C, NUL) == SHAPE


def test_gemm_validation(lib):
    f = lib.w4a4_gemm
    args = [A, B, C, D, 64, 256, 256, 64, NUL, NUL, 0, NUL, E, NUL, NUL]
    bad = list(args); bad[4] = 0
    assert f(*bad) == SHAPE
    bad = list(args); bad[5] = 12                      # N not a multiple of 8
    assert f(*bad) == SHAPE
    bad = list(args); bad[6] = 320
    assert f(*bad) == SHAPE
    bad = list(args); bad[12] = NUL                    # no output
    assert f(*bad) == INVALID
    bad = list(args); bad[10] = 16                     # rank without T / L2
    assert f(*bad) == INVALID
    bad = list(args); bad[11] = ODD                    # misaligned bias
    assert f(*bad) == MISALIGNED
    bad = list(args); bad[13] = ODD                    # misaligned debug output
    assert f(*bad) == MISALIGNED
    assert lib.w8a8_gemm(A, B, C, D, 64, 4, 256, 128, NUL, E, NUL, NUL) == SHAPE


def test_mlp_workspace_and_validation(lib):
    M, D, H = 4608, 3072, 12288
    need = lib.w4a4_mlp_workspace_bytes(M, D, H, 128, 128)
    up = lib.w4a4_workspace_bytes(M, D, 128)
    down = lib.w4a4_workspace_bytes(M, H, 128)
    assert need == up + M * H * 2 + down      # every part already 256-aligned here
    assert lib.w4a4_mlp_workspace_bytes(0, D, H, 0, 0) == 0
    f = lib.w4a4_mlp
    args = [A, 64, 256, 512, 128, B, C, NUL, NUL, 0, NUL, D, E, NUL, NUL, 0, NUL, E, E,
            lib.w4a4_mlp_workspace_bytes(64, 256, 512, 0, 0), NUL]
    bad = list(args); bad[5] = NUL                       # no up weights
    assert f(*bad) == INVALID
    bad = list(args); bad[19] = 1                         # workspace too small
    assert f(*bad) == WORKSPACE
    bad = list(args); bad[0] = 0                          # no input  (NULL)
    assert f(*bad) == INVALID
    g = lib.w4a4_gemm_gelu
    assert g(A, B, C, D, 64, 12, 256, 64, NUL, NUL, 0, NUL, E, NUL, NUL) == SHAPE
    assert lib.w4a4_linear_gelu(A, B, C, 64, 256, 256, 64, NUL, NUL, 0, NUL, D, E, 1, NUL) == WORKSPACE


def test_bake_lora_sr_validation(lib):
    f = lib.w4a4_bake_lora_sr
    args = [A, B, C, 16, 0.5, 64, 256, 128, 7, D, E, E, NUL]
    bad = list(args); bad[2] = NUL
    assert f(*bad) == INVALID
    bad = list(args); bad[3] = 0                      # no LoRA rank
    assert f(*bad) == SHAPE
    bad = list(args); bad[6] = 320                    # K not a multiple of 128
    assert f(*bad) == SHAPE
    bad = list(args); bad[9] = ODD
    assert f(*bad) == MISALIGNED


def test_lora_merge_validation(lib):
    f = lib.w4a4_lora_merge
    args = [A, B, 16, C, D, 32, 0.5, 256, 512, E, E, NUL]
    bad = list(args); bad[3] = NUL                      # no LoRA down matrix
    assert f(*bad) == INVALID
    bad = list(args); bad[0] = NUL                      # rank > 0 without L1
    assert f(*bad) == INVALID
    bad = list(args); bad[5] = 8                        # LoRA rank not a multiple of 16
    assert f(*bad) == SHAPE
    bad = list(args); bad[5] = 256                      # combined rank above 256
    assert f(*bad) == SHAPE
    bad = list(args); bad[8] = 12                       # N not a multiple of 8
    assert f(*bad) == SHAPE
    bad = list(args); bad[9] = ODD
    assert f(*bad) == MISALIGNED
    assert f(NUL, NUL, 0, C, D, 32, 0.5, 256, 512, ODD, E, NUL) == MISALIGNED   # r = 0 needs no L1 / L2


def test_w4a8_validation(lib):
    # quantize: the zero-point output is required
    assert lib.w4a8_quantize_weights(A, 64, 256, 64, B, C, NUL, NUL) == INVALID
    assert lib.w4a8_quantize_weights(A, 64, 320, 64, B, C, D, NUL) == SHAPE
    assert lib.w4a8_quantize_weights(ODD, 64, 256, 64, B, C, D, NUL) == MISALIGNED
    g = lib.w4a8_gemm
    args = [A, B, C, D, E, 64, 256, 256, 128, NUL, E, NUL, NUL]
    bad = list(args); bad[4] = NUL                     # no zero points
    assert g(*bad) == INVALID
    bad = list(args); bad[6] = 12                      # N not a multiple of 8
    assert g(*bad) == SHAPE
    bad = list(args); bad[8] = 32                      # unsupported group
    assert g(*bad) == SHAPE
    bad = list(args); bad[2] = ODD                     # misaligned codes
    assert g(*bad) == MISALIGNED
    assert lib.w4a8_workspace_bytes(5, 256) == lib.w8a8_workspace_bytes(5, 256)
    need = lib.w4a8_workspace_bytes(16, 256)
    assert lib.w4a8_linear(A, B, C, D, 16, 256, 256, 128, NUL, E, E, need - 1, NUL) == WORKSPACE
    assert lib.w4a8_linear(A, B, C, NUL, 16, 256, 256, 128, NUL, E, E, need, NUL) == INVALID


def test_linear_workspace_rules(lib):
    need = lib.w4a4_workspace_bytes(4608, 3072, 0)
    assert need == 4608 * 1536 + 4608 * 4 + 0
    assert lib.w4a4_workspace_bytes(3, 256, 16) == 512 + 256 + 256   # 384 B codes, 12 B scales, 96 B T
    assert lib.w4a4_workspace_bytes(0, 256, 0) == 0
    assert lib.w8a8_workspace_bytes(5, 256) == 1280 + 256
    f = lib.w4a4_linear
    args = [A, B, C, 4608, 3072, 3072, 128, NUL, NUL, 0, NUL, D, E, need, NUL]
    bad = list(args); bad[13] = need - 1
    assert f(*bad) == WORKSPACE
    bad = list(args); bad[12] = NUL
    assert f(*bad) == WORKSPACE
    bad = list(args); bad[12] = ctypes.c_void_p(0x50010)   # not 256-byte aligned
    assert f(*bad) == WORKSPACE
    bad = list(args); bad[9] = 64                          # rank without L1/L2
    assert f(*bad) == INVALID
    g = lib.w8a8_linear
    need8 = lib.w8a8_workspace_bytes(16, 256)
    assert g(A, B, C, 16, 256, 256, 128, NUL, D, E, need8 - 1, NUL) == WORKSPACE


def _cuda_visible():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.mark.skipif(_cuda_visible(), reason="only meaningful on a host without a GPU")
def test_valid_call_without_gpu_fails_loudly(lib):
    # all arguments valid: the call reaches the device check and must report
    # that no CUDA device can run it (there is no CPU fallback)
    assert lib.w4a4_quantize_weights(A, 64, 256, 64, B, C, NUL) in (CUDA, DEVICE)
    with pytest.raises(w4.W4A4Error):
        w4._check("w4a4_quantize_weights", lib.w4a4_quantize_weights(A, 64, 256, 64, B, C, NUL))


def test_selftest_wait_timeout_validation(lib):
    f = lib.w4a4_selftest_wait_timeout
    assert f(NUL, B, 64, 256, 16, C, 1000, NUL) == INVALID
    assert f(A, NUL, 64, 256, 16, C, 1000, NUL) == INVALID
    assert f(A, B, 64, 256, 16, NUL, 1000, NUL) == INVALID
    assert f(A, B, 64, 256, 16, C, 0, NUL) == INVALID          # no wait limit
    assert f(A, B, 64, 256, 16, C, 2000000, NUL) == INVALID    # over one second
    assert f(A, B, 64, 256, 0, C, 1000, NUL) == SHAPE          # needs a low-rank branch
    assert f(A, B, 64, 256, 24, C, 1000, NUL) == SHAPE         # rank not a multiple of 16
    assert f(A, B, 0, 256, 16, C, 1000, NUL) == SHAPE
    assert f(A, B, 64, 200, 16, C, 1000, NUL) == SHAPE
    assert f(ODD, B, 64, 256, 16, C, 1000, NUL) == MISALIGNED


def test_device_error_bits_match_the_header():
    text = open(HEADER).read()
    bits = dict(re.findall(r"#define W4A4_DEVERR_(\w+) (\d+)u", text))
    assert {k: int(v) for k, v in bits.items()} == {
        "WAIT_OPERANDS": w4.DEVERR_WAIT_OPERANDS, "WAIT_SLOT": w4.DEVERR_WAIT_SLOT,
        "WAIT_ACCUM": w4.DEVERR_WAIT_ACCUM, "WAIT_DRAIN": w4.DEVERR_WAIT_DRAIN}


def test_launch_plan_cache_under_host_threads(lib):
    """The launch-plan cache hands every thread the plan of the shape it asked
    for while other threads insert and evict other shapes (no CUDA call)."""
    import concurrent.futures as cf
    import random
    shapes = [(m, k, g) for m in (1, 2, 37, 256, 1000, 4608, 9216, 16384)
              for k in (256, 3072, 12288) for g in (64, 128)]
    expect = {sh: w4.w4a4_plan_rotate_quantize(*sh, cached=False) for sh in shapes}
    assert expect[(4608, 3072, 128)] == (4, 96, 2 * 4 * 3072 * 2 + 1024, 592)

    def worker(seed):
        rnd = random.Random(seed)
        bad = 0
        for _ in range(4000):
            sh = rnd.choice(shapes)
            if w4.w4a4_plan_rotate_quantize(*sh, cached=True) != expect[sh]:
                bad += 1
        return bad

    with cf.ThreadPoolExecutor(8) as ex:
        assert sum(ex.map(worker, range(8))) == 0


@pytest.mark.parametrize("M,N,K,rank,kw,expect", [
    (256, 3072, 3072, 0, {}, 4),          # 12 tiles: four pairs per tile fill 48 of 74 pairs
    (512, 3072, 3072, 0, {}, 2),          # 24 tiles: 4 x 24 > 74, 2 x 24 fits
    (4608, 3072, 3072, 0, {}, 1),         # 216 tiles: the persistent form
    (40, 8, 3072, 0, {}, 4),              # one tile
    (64, 256, 256, 0, {}, 1),             # two k-blocks: no slice would keep two
    (1, 3072, 512, 0, {}, 2),             # four k-blocks: two slices of two
    (256, 3072, 12288, 16, {}, 4),        # small rank on a long K range
    (256, 3072, 12288, 32, {}, 4),
    (256, 3072, 12288, 64, {}, 1),        # larger ranks keep the tensor-core low-rank MMA
    (256, 3072, 3072, 16, {}, 1),         # short K range with a low-rank branch
    (256, 3072, 3072, 0, {"clusters_of_8": 8}, 2),                      # 12 clusters of 8 do not fit
    (256, 3072, 3072, 0, {"clusters_of_8": 8, "clusters_of_4": 8}, 1),  # nor 12 of 4
    (256, 3072, 3072, 0, {"sms": 40}, 1),                               # too few SMs for any split
])
def test_plan_gemm_split(M, N, K, rank, kw, expect):
    """The GEMM's split-K decision, host only: the same function the
    launchers call with the device's occupancy figures."""
    assert w4.w4a4_plan_gemm_split(M, N, K, rank, **kw) == expect


def test_plan_gemm_split_validation(lib):
    import ctypes
    out = ctypes.c_int(0)
    f = lib.w4a4_plan_gemm_split
    assert f(256, 3072, 3072, 0, 148, 16, 32, None) == 1                  # W4A4_ERR_INVALID_ARG
    assert f(256, 3070, 3072, 0, 148, 16, 32, ctypes.byref(out)) == 2     # N not a multiple of 8
    assert f(256, 3072, 3000, 0, 148, 16, 32, ctypes.byref(out)) == 2     # K not a multiple of 128
    assert f(256, 3072, 3072, 20, 148, 16, 32, ctypes.byref(out)) == 2    # rank not a multiple of 16
    assert f(0, 3072, 3072, 0, 148, 16, 32, ctypes.byref(out)) == 2       # empty M
    assert f(256, 3072, 3072, 0, 148, 16, 32, ctypes.byref(out)) == 0 and out.value == 4
