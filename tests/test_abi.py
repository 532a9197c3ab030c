"""The C ABI library loads, exports every entry point its header declares,
and rejects bad arguments on the host before touching the GPU (these calls
need no GPU). Also checks that the product path never falls back to the CPU."""
import ctypes
import os
import re

import pytest

from moe_gemm_token_b200 import build as libbuild
from moe_gemm_token_b200 import metis

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return metis.load()


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"METIS_API\s+[\w\s\*]+?\b(metis_\w+)\s*\(", text)
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    dyn = os.popen(f"nm -D --defined-only {metis.LIB_PATH}").read()
    for n in names:
        assert re.search(rf"\bT {n}\b", dyn), n


def test_build_targets_sm100a_only():
    assert libbuild.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert "--use_fast_math" not in libbuild.FLAGS


def test_version(lib):
    assert metis.metis_version() == 100


def _rc(fn, *args):
    return fn(*args)


def test_host_validation_without_gpu(lib):
    p = ctypes.c_void_p(0x1000)
    null = None
    # quantizer: K not a multiple of 8, bad leading dimensions
    assert lib.metis_quant_fp8_per_token(p, 4, 12, 12, p, 16, p, null) == metis.METIS_ERR_INVALID_ARG
    assert b"K % 8" in lib.metis_last_error()
    assert lib.metis_quant_fp8_per_token(p, 4, 16, 8, p, 16, p, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_quant_fp8_per_token(p, 4, 16, 16, p, 20, p, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_quant_fp8_per_token(p, 0, 16, 16, p, 16, p, null) == metis.METIS_OK  # nothing to do
    assert lib.metis_quant_fp8_per_token(null, 4, 16, 16, p, 16, p, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_quant_fp8_per_token(ctypes.c_void_p(0x1008), 4, 16, 16, p, 16, p, null) == \
        metis.METIS_ERR_INVALID_ARG  # misaligned x
    assert lib.metis_quant_fp8_per_channel(p, 4, 6, 8, p, 16, p, null) == metis.METIS_ERR_INVALID_ARG
    # GEMM: K % 16, N % 8, bad kind
    assert lib.metis_fp8_gemm(p, 0, p, p, p, p, 16, 512, 40, null, 0, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_fp8_gemm(p, 0, p, p, p, p, 16, 500, 256, null, 0, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_fp8_gemm(p, 7, p, p, p, p, 16, 512, 256, null, 0, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_fp8_gemm(p, 0, p, p, p, p, 0, 512, 256, null, 0, null) == metis.METIS_OK
    # fused quantization (BF16 A): a workspace of align256(4 * M) bytes, 16-byte aligned
    need = lib.metis_workspace_size(metis.METIS_OP_FP8_GEMM_FUSED, 300, 512, 256, 0, 0)
    assert need == 1280
    assert lib.metis_fp8_gemm(p, 1, p, p, p, p, 300, 512, 256, null, 0, null) == metis.METIS_ERR_INVALID_ARG
    assert b"workspace" in lib.metis_last_error()
    assert lib.metis_fp8_gemm(p, 1, p, p, p, p, 300, 512, 256, p, need - 4, null) == \
        metis.METIS_ERR_INVALID_ARG
    assert lib.metis_fp8_gemm(p, 1, p, p, p, p, 300, 512, 256, ctypes.c_void_p(0x1004), need,
                              null) == metis.METIS_ERR_INVALID_ARG
    # W8A16: M = 0; M > 8 needs N % 8; K too large for the decode kernel
    assert lib.metis_w8a16_gemm(p, p, p, p, 0, 128, 256, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_w8a16_gemm(p, p, p, p, 9, 100, 256, null) == metis.METIS_ERR_INVALID_ARG
    assert b"N % 8" in lib.metis_last_error()
    assert lib.metis_w8a16_gemm(p, p, p, p, 9, 128, 250, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_w8a16_gemm(p, p, p, p, 4, 128, 16384, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_w8a16_gemm(p, p, p, p, 4, 128, 264, null) == metis.METIS_ERR_INVALID_ARG
    # W8A16 through widened weights: N % 8, K % 16, the workspace of 2 N K bytes
    need_w = lib.metis_workspace_size(metis.METIS_OP_W8A16_WIDENED, 300, 6144, 2048, 0, 0)
    assert need_w == 2 * 6144 * 2048
    assert lib.metis_workspace_size(metis.METIS_OP_W8A16_WIDENED, 0, 6144, 2048, 0, 0) == 0
    assert lib.metis_w8a16_gemm_widened(p, p, p, p, 300, 100, 256, p, 1 << 30, null) == \
        metis.METIS_ERR_INVALID_ARG
    assert lib.metis_w8a16_gemm_widened(p, p, p, p, 300, 128, 250, p, 1 << 30, null) == \
        metis.METIS_ERR_INVALID_ARG
    assert lib.metis_w8a16_gemm_widened(p, p, p, p, 300, 6144, 2048, p, need_w - 16, null) == \
        metis.METIS_ERR_INVALID_ARG
    assert b"workspace" in lib.metis_last_error()
    assert lib.metis_w8a16_gemm_widened(p, p, p, p, 300, 6144, 2048, ctypes.c_void_p(0x1008), need_w,
                                        null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_w8a16_gemm_widened(p, p, p, p, 0, 6144, 2048, p, 0, null) == metis.METIS_OK
    # MoE: activation, topk > E, H % 16, small workspace
    assert lib.metis_moe_fp8_grouped_gemm(p, p, p, 8, 2, 4, 64, 32, p, p, p, p, 1, p, p, 1 << 30,
                                          null) == metis.METIS_ERR_UNSUPPORTED
    assert lib.metis_moe_fp8_grouped_gemm(p, p, p, 8, 5, 4, 64, 32, p, p, p, p, 0, p, p, 1 << 30,
                                          null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_moe_fp8_grouped_gemm(p, p, p, 8, 2, 4, 72, 32, p, p, p, p, 0, p, p, 1 << 30,
                                          null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_moe_fp8_grouped_gemm(p, p, p, 8, 2, 4, 64, 32, p, p, p, p, 0, p, p, 16,
                                          null) == metis.METIS_ERR_INVALID_ARG
    assert b"workspace" in lib.metis_last_error()
    # allocation-free routed layer: the same shape checks first (an unsupported
    # activation is reported as such, absurd T is rejected before any size is
    # computed), then y is required, then the built-in scratch bounds the size
    na = lib.metis_moe_fp8_grouped_gemm_noalloc
    assert na(p, p, p, 4096, 8, 64, 2048, 1024, p, p, p, p, 1, p, null) == metis.METIS_ERR_UNSUPPORTED
    assert na(p, p, p, 8, 5, 4, 64, 32, p, p, p, p, 0, p, null) == metis.METIS_ERR_INVALID_ARG
    assert na(p, p, p, 1 << 40, 8, 64, 2048, 1024, p, p, p, p, 0, p, null) == metis.METIS_ERR_INVALID_ARG
    assert na(p, p, p, 0, 8, 64, 2048, 1024, p, p, p, p, 0, null, null) == metis.METIS_OK  # nothing to do
    assert na(p, p, p, 16, 8, 64, 2048, 1024, p, p, p, p, 0, null, null) == metis.METIS_ERR_INVALID_ARG
    assert b"y is required" in lib.metis_last_error()
    assert na(p, p, p, 4096, 8, 64, 2048, 1024, p, p, p, p, 0, p, null) == metis.METIS_ERR_INVALID_ARG
    assert b"16 MiB" in lib.metis_last_error()
    # watchdog self-test: the limit must be 1 .. 1e9 ns
    assert lib.metis_watchdog_selftest(0, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_watchdog_selftest(2000000000, null) == metis.METIS_ERR_INVALID_ARG
    # router top-k: topk > E, E > 1024, topk > 32
    assert lib.metis_moe_route_topk(p, null, 8, 4, 5, p, p, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_moe_route_topk(p, null, 8, 1025, 4, p, p, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_moe_route_topk(p, null, 8, 64, 33, p, p, null) == metis.METIS_ERR_INVALID_ARG
    assert lib.metis_moe_route_topk(p, null, 0, 64, 8, p, p, null) == metis.METIS_OK
    # dispatch: the default maths for M > 8 validates like metis_w8a16_gemm
    assert lib.metis_linear(p, p, p, p, 64, 100, 256, 0, p, p, 1 << 20, null) == metis.METIS_ERR_INVALID_ARG
    # fast-math dispatch needs room for the codes of x
    assert lib.metis_workspace_size(metis.METIS_OP_LINEAR, 64, 128, 256, 0, 0) == 64 * 256
    assert lib.metis_workspace_size(metis.METIS_OP_LINEAR, 8, 128, 256, 0, 0) == 0
    assert lib.metis_linear(p, p, p, p, 64, 128, 256, 1, p, p, 64 * 256 - 16, null) == \
        metis.METIS_ERR_INVALID_ARG
    assert b"workspace" in lib.metis_last_error()


def test_valid_call_without_gpu_fails_loudly(lib):
    """No CPU fallback: a well-formed call on a machine without a GPU returns
    METIS_ERR_CUDA instead of computing anything."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    p = ctypes.c_void_p(0x1000)
    rc = lib.metis_quant_fp8_per_token(p, 4, 16, 16, p, 16, p, None)
    assert rc == metis.METIS_ERR_CUDA
    assert lib.metis_last_error()


def test_workspace_layout(lib):
    T, k, E, H, I = 4096, 8, 64, 2048, 1024
    total = metis.metis_workspace_size(metis.METIS_OP_MOE, T, I, H, k, E)
    offs = [metis.metis_moe_workspace_offset(r, T, k, E, H, I) for r in range(10)]
    assert offs[0] == 0 and all(o % 256 == 0 for o in offs)
    assert all(b > a for a, b in zip(offs, offs[1:]))
    S = T * k
    sizes = [4 * E, 4 * (E + 1), 4 * S, 4 * S, S * H, 4 * S, 2 * S * I, S * I, 4 * S, 2 * S * H]
    for o, s, nxt in zip(offs, sizes, offs[1:] + [total]):
        assert o + s <= nxt
    assert metis.metis_moe_workspace_offset(10, T, k, E, H, I) == -1
    assert metis.metis_workspace_size(metis.METIS_OP_FP8_GEMM_FUSED, 4096, 2048, 2048) >= 4 * 4096
    assert metis.metis_workspace_size(metis.METIS_OP_FP8_GEMM, 4096, 2048, 2048) == 0


def test_nvfp4_host_validation_without_gpu(lib):
    p = ctypes.c_void_p(0x1000)
    null = None
    E = metis.METIS_ERR_INVALID_ARG
    # quantizer: K not a multiple of 64, bad kind, rows_per_scale not dividing R
    assert lib.metis_quant_nvfp4(p, metis.METIS_A_BF16, 4, 96, 96, 1, p, p, 0, p, null) == E
    assert b"K" in lib.metis_last_error()
    assert lib.metis_quant_nvfp4(p, 7, 4, 64, 64, 1, p, p, 0, p, null) == E
    assert lib.metis_quant_nvfp4(p, metis.METIS_A_F32, 6, 64, 64, 4, p, p, 0, p, null) == E
    assert lib.metis_quant_nvfp4(p, metis.METIS_A_BF16, 4, 64, 64, 1, p, p, 9, p, null) == E
    assert lib.metis_quant_nvfp4(p, metis.METIS_A_BF16, 0, 64, 64, 1, p, p, 0, p, null) == metis.METIS_OK
    # scale re-layout: K % 64, overlap
    assert lib.metis_nvfp4_scales_to_tiled(p, 4, 80, p, null) == E
    assert lib.metis_nvfp4_scales_to_tiled(p, 128, 64, ctypes.c_void_p(0x1100), null) == E
    assert b"overlap" in lib.metis_last_error()
    # GEMM: N not a multiple of 128, K not a multiple of 64, misaligned y
    assert lib.metis_nvfp4_gemm(p, p, p, p, p, p, p, 4, 200, 256, null) == E
    assert lib.metis_nvfp4_gemm(p, p, p, p, p, p, p, 4, 256, 96, null) == E
    assert lib.metis_nvfp4_gemm(p, p, p, p, p, p, ctypes.c_void_p(0x1008), 4, 256, 256, null) == E
    assert lib.metis_nvfp4_gemm(p, p, p, p, p, p, p, 0, 256, 256, null) == metis.METIS_OK
    # routed experts: H or I not a multiple of 128, topk > E, small workspace
    args = lambda T, k, Ex, H, I, ws: (p, p, p, T, k, Ex, H, I, p, p, p, p, p, p, 0, p, p, ws, null)
    assert lib.metis_moe_nvfp4_grouped_gemm(*args(8, 2, 8, 192, 256, 1 << 30)) == E
    assert lib.metis_moe_nvfp4_grouped_gemm(*args(8, 9, 8, 256, 256, 1 << 30)) == E
    need = metis.metis_workspace_size(metis.METIS_OP_MOE_NVFP4, 8, 256, 256, 2, 8)
    assert lib.metis_moe_nvfp4_grouped_gemm(*args(8, 2, 8, 256, 256, need - 256)) == E
    assert b"workspace" in lib.metis_last_error()
    assert lib.metis_moe_nvfp4_grouped_gemm(*args(0, 2, 8, 256, 256, 0)) == metis.METIS_OK


def test_nvfp4_workspace_layout(lib):
    T, k, E, H, I = 4096, 8, 64, 2048, 1024
    total = metis.metis_workspace_size(metis.METIS_OP_MOE_NVFP4, T, I, H, k, E)
    offs = [metis.metis_moe_nvfp4_workspace_offset(r, T, k, E, H, I) for r in range(12)]
    S = T * k
    Sp = (S + 127 * E + 127) // 128 * 128
    sizes = [4 * E, 4 * (E + 1), 4 * S, 4 * Sp, Sp * H // 2, Sp * H // 16, 4 * Sp, 2 * Sp * I,
             Sp * I // 2, Sp * I // 16, 4 * Sp, 2 * Sp * H]
    assert offs[0] == 0 and all(o % 256 == 0 for o in offs)
    for o, s, nxt in zip(offs, sizes, offs[1:] + [total]):
        assert o + s <= nxt
    assert metis.metis_moe_nvfp4_workspace_offset(12, T, k, E, H, I) == -1


def test_shared_expert_host_validation_without_gpu(lib):
    p = ctypes.c_void_p(0x1000)
    null = None
    E = metis.METIS_ERR_INVALID_ARG
    # BF16 GEMM: N or K not a multiple of 8, misaligned y, M = 0 is a no-op
    assert lib.metis_bf16_gemm(p, p, p, 4, 12, 16, null) == E
    assert lib.metis_bf16_gemm(p, p, p, 4, 16, 12, null) == E
    assert lib.metis_bf16_gemm(p, p, ctypes.c_void_p(0x1008), 4, 16, 16, null) == E
    assert lib.metis_bf16_gemm(p, p, p, 0, 16, 16, null) == metis.METIS_OK
    # fused shared combine: topk > 8, H not a multiple of 16, workspace too small
    need = metis.metis_workspace_size(metis.METIS_OP_SHARED, 8, 64, 128, 2, 0)
    assert need == 8 * 64 * 2 or need >= 8 * 64 * 2
    args = lambda T, H, Is, k, ws: (p, T, H, Is, p, p, p, p, p, k, p, p, ws, null)
    assert lib.metis_moe_shared_fused_combine(*args(8, 128, 64, 9, need)) == E
    assert lib.metis_moe_shared_fused_combine(*args(8, 120, 64, 2, need)) == E
    assert lib.metis_moe_shared_fused_combine(*args(8, 128, 64, 2, need - 16)) == E
    assert b"workspace" in lib.metis_last_error()
    assert lib.metis_moe_shared_fused_combine(*args(0, 128, 64, 2, 0)) == metis.METIS_OK
