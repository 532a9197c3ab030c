"""Thin Python binding of libmetis_fp8 (the C ABI in ``include/metis_fp8.h``).

Every function here has the name of the C entry point it calls and only
marshals arguments: torch CUDA tensors become device pointers, shapes become
sizes, the current torch stream becomes the ``cudaStream_t``. All arithmetic
runs in the library's CUDA kernels. There is no fallback: if the library is
missing, :func:`load` raises.

BF16 tensors may be ``torch.bfloat16`` or ``torch.int16``/``uint16`` bit
patterns; E4M3 tensors ``torch.uint8`` or ``torch.float8_e4m3fn``.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmetis_fp8.so")

METIS_OK = 0
METIS_ERR_INVALID_ARG = -1
METIS_ERR_UNSUPPORTED = -2
METIS_ERR_CUDA = -3
METIS_ERR_TIMEOUT = -4

METIS_A_E4M3 = 0
METIS_A_BF16 = 1
METIS_ACT_NONE = 0
METIS_OP_FP8_GEMM = 0
METIS_OP_FP8_GEMM_FUSED = 1
METIS_OP_W8A16 = 2
METIS_OP_MOE = 3
METIS_OP_LINEAR = 4
METIS_OP_MOE_NVFP4 = 5
METIS_OP_SHARED = 6
METIS_OP_W8A16_WIDENED = 7
METIS_A_F32 = 2
METIS_SF_ROWMAJOR = 0
METIS_SF_TILED = 1

MOE_WS = dict(COUNTS=0, OFFSETS=1, SLOT_TO_ROW=2, ROW_TO_SLOT=3, AQ=4, SA=5, H=6, HQ=7, SH=8,
              O=9)

MOE4_WS = dict(COUNTS=0, OFFSETS=1, SLOT_TO_ROW=2, ROW_TO_SLOT=3, AQ=4, SFA=5, GA=6, H=7, HQ=8,
               SFH=9, GH=10, O=11)

_lib = None


class MetisError(RuntimeError):
    def __init__(self, name, code, msg):
        super().__init__(f"{name} returned {code}: {msg}")
        self.code = code


def load():
    """Loads libmetis_fp8.so (built in-tree by ``moe_gemm_token_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m moe_gemm_token_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    sz = ctypes.c_size_t
    sig = {
        "metis_version": ([], i32),
        "metis_last_error": ([], ctypes.c_char_p),
        "metis_check_device_status": ([p, i32], i32),
        "metis_set_watchdog_ns": ([ctypes.c_uint64], i32),
        "metis_watchdog_selftest": ([ctypes.c_uint64, p], i32),
        "metis_quant_fp8_per_token": ([p, i64, i64, i64, p, i64, p, p], i32),
        "metis_quant_fp8_per_channel": ([p, i64, i64, i64, p, i64, p, p], i32),
        "metis_fp8_gemm": ([p, i32, p, p, p, p, i64, i64, i64, p, sz, p], i32),
        "metis_w8a16_gemm": ([p, p, p, p, i64, i64, i64, p], i32),
        "metis_w8a16_gemm_widened": ([p, p, p, p, i64, i64, i64, p, sz, p], i32),
        "metis_moe_route_topk": ([p, p, i64, i64, i64, p, p, p], i32),
        "metis_moe_fp8_grouped_gemm": ([p, p, p, i64, i64, i64, i64, i64, p, p, p, p, i32, p, p,
                                        sz, p], i32),
        "metis_moe_fp8_grouped_gemm_noalloc": ([p, p, p, i64, i64, i64, i64, i64, p, p, p, p,
                                                i32, p, p], i32),
        "metis_workspace_size": ([i32, i64, i64, i64, i64, i64], sz),
        "metis_moe_workspace_offset": ([i32, i64, i64, i64, i64, i64], i64),
        "metis_linear": ([p, p, p, p, i64, i64, i64, i32, p, p, sz, p], i32),
        "metis_quant_nvfp4": ([p, i32, i64, i64, i64, i64, p, p, i32, p, p], i32),
        "metis_nvfp4_scales_to_tiled": ([p, i64, i64, p, p], i32),
        "metis_nvfp4_gemm": ([p, p, p, p, p, p, p, i64, i64, i64, p], i32),
        "metis_moe_nvfp4_grouped_gemm": ([p, p, p, i64, i64, i64, i64, i64, p, p, p, p, p, p, i32,
                                          p, p, sz, p], i32),
        "metis_moe_nvfp4_workspace_offset": ([i32, i64, i64, i64, i64, i64], i64),
        "metis_bf16_gemm": ([p, p, p, i64, i64, i64, p], i32),
        "metis_moe_shared_fused_combine": ([p, i64, i64, i64, p, p, p, p, p, i64, p, p, sz, p], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(name, rc):
    if rc != METIS_OK:
        raise MetisError(name, rc, load().metis_last_error().decode())
    return rc


def _rows(t):
    return t.shape[0], t.shape[1], t.stride(0)


def metis_version():
    return load().metis_version()


def metis_check_device_status(stream=None, clear=True):
    """Synchronises the stream and returns the sticky device status (0 = OK)."""
    return load().metis_check_device_status(_s(stream), int(bool(clear)))


def metis_watchdog_selftest(limit_ns, stream=None):
    """Launches a wait that nothing satisfies, bounded by limit_ns (see the header)."""
    return _check("metis_watchdog_selftest", load().metis_watchdog_selftest(int(limit_ns), _s(stream)))


def metis_set_watchdog_ns(ns):
    return _check("metis_set_watchdog_ns", load().metis_set_watchdog_ns(int(ns)))


def metis_quant_fp8_per_token(x, xq, s_tok, stream=None):
    """x [M, K] BF16 -> xq [M, K] E4M3 codes, s_tok [M] FP32."""
    M, K, ldx = _rows(x)
    return _check("metis_quant_fp8_per_token", load().metis_quant_fp8_per_token(
        _p(x), M, K, ldx, _p(xq), xq.stride(0), _p(s_tok), _s(stream)))


def metis_quant_fp8_per_channel(w, wq, s_w, stream=None):
    """w [N, K] FP32 -> wq [N, K] E4M3 codes, s_w [N] FP32."""
    N, K, ldw = _rows(w)
    return _check("metis_quant_fp8_per_channel", load().metis_quant_fp8_per_channel(
        _p(w), N, K, ldw, _p(wq), wq.stride(0), _p(s_w), _s(stream)))


def metis_fp8_gemm(a, a_kind, s_tok, wq, s_w, y, workspace=None, stream=None):
    """y [M, N] = W8A8(a, wq); a is E4M3 (a_kind 0) or BF16 (a_kind 1, fused quantization)."""
    M, K = a.shape
    N = wq.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return _check("metis_fp8_gemm", load().metis_fp8_gemm(
        _p(a), int(a_kind), _p(s_tok), _p(wq), _p(s_w), _p(y), M, N, K, _p(workspace), ws_bytes,
        _s(stream)))


def metis_w8a16_gemm(x, wq, s_w, y, stream=None):
    """y [M, N] = W8A16(x, wq): the default maths (decode kernel for M <= 8,
    tensor-core kernel for M > 8)."""
    M, K = x.shape
    N = wq.shape[0]
    return _check("metis_w8a16_gemm", load().metis_w8a16_gemm(
        _p(x), _p(wq), _p(s_w), _p(y), M, N, K, _s(stream)))


def metis_w8a16_gemm_widened(x, wq, s_w, y, workspace, stream=None):
    """y [M, N] = W8A16(x, wq) with the weights widened to BF16 into `workspace`
    first (metis_workspace_size(METIS_OP_W8A16_WIDENED, M, N, K) bytes)."""
    M, K = x.shape
    N = wq.shape[0]
    ws_bytes = workspace.numel() * workspace.element_size()
    return _check("metis_w8a16_gemm_widened", load().metis_w8a16_gemm_widened(
        _p(x), _p(wq), _p(s_w), _p(y), M, N, K, _p(workspace), ws_bytes, _s(stream)))


def metis_moe_route_topk(logits, topk_ids, topk_w, bias=None, stream=None):
    """Router top-k: logits [T, E] FP32 (+ bias [E]) -> topk_ids [T, k], topk_w [T, k]."""
    T, E = logits.shape
    k = topk_ids.shape[1]
    return _check("metis_moe_route_topk", load().metis_moe_route_topk(
        _p(logits), _p(bias), T, E, k, _p(topk_ids), _p(topk_w), _s(stream)))


def metis_moe_fp8_grouped_gemm(x, topk_ids, topk_w, w_up, s_up, w_down, s_down, y, workspace,
                               act=METIS_ACT_NONE, stream=None):
    """Routed-expert W8A8 layer; see the C header for shapes."""
    T, H = x.shape
    topk = topk_ids.shape[1]
    E, I, H2 = w_up.shape
    assert H2 == H
    ws_bytes = workspace.numel() * workspace.element_size()
    return _check("metis_moe_fp8_grouped_gemm", load().metis_moe_fp8_grouped_gemm(
        _p(x), _p(topk_ids), _p(topk_w), T, topk, E, H, I, _p(w_up), _p(s_up), _p(w_down),
        _p(s_down), int(act), _p(y), _p(workspace), ws_bytes, _s(stream)))


def metis_moe_fp8_grouped_gemm_noalloc(x, topk_ids, topk_w, w_up, s_up, w_down, s_down, y,
                                       act=METIS_ACT_NONE, stream=None):
    """Routed-expert W8A8 layer without a caller workspace (built-in 16 MiB scratch)."""
    T, H = x.shape
    topk = topk_ids.shape[1]
    E, I, H2 = w_up.shape
    assert H2 == H
    return _check("metis_moe_fp8_grouped_gemm_noalloc", load().metis_moe_fp8_grouped_gemm_noalloc(
        _p(x), _p(topk_ids), _p(topk_w), T, topk, E, H, I, _p(w_up), _p(s_up), _p(w_down),
        _p(s_down), int(act), _p(y), _s(stream)))


def metis_workspace_size(op, m_or_t, n_or_i, k_or_h, topk=0, num_experts=0):
    return int(load().metis_workspace_size(int(op), int(m_or_t), int(n_or_i), int(k_or_h),
                                           int(topk), int(num_experts)))


def metis_moe_workspace_offset(region, T, topk, E, H, I):
    if isinstance(region, str):
        region = MOE_WS[region]
    return int(load().metis_moe_workspace_offset(int(region), int(T), int(topk), int(E), int(H),
                                                 int(I)))


def metis_linear(x, wq, s_w, y, fast_math=True, s_tok=None, workspace=None, stream=None):
    """Dispatch rule: M <= 8 -> W8A16; otherwise W8A8 with fast_math (per-token
    quantizer into `workspace`, then the E4M3 GEMM) and W8A16 without (the
    widened-weights GEMM when M >= 2048 and `workspace` holds the BF16 weights)."""
    M, K = x.shape
    N = wq.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return _check("metis_linear", load().metis_linear(
        _p(x), _p(wq), _p(s_w), _p(y), M, N, K, int(bool(fast_math)), _p(s_tok), _p(workspace),
        ws_bytes, _s(stream)))


# ------------------------------------------------------------------ NVFP4

def metis_quant_nvfp4(x, q, sf, g, rows_per_scale=1, tiled=False, stream=None):
    """x [R, K] BF16 (or FP32) -> q [R, K/2] packed E2M1 codes, sf block scales
    (row-major [R, K/16], or tiled), g [R / rows_per_scale] global scales."""
    R, K, ldx = _rows(x)
    kind = METIS_A_F32 if x.dtype == torch.float32 else METIS_A_BF16
    return _check("metis_quant_nvfp4", load().metis_quant_nvfp4(
        _p(x), kind, R, K, ldx, int(rows_per_scale), _p(q), _p(sf),
        METIS_SF_TILED if tiled else METIS_SF_ROWMAJOR, _p(g), _s(stream)))


def metis_nvfp4_scales_to_tiled(sf, sf_tiled, stream=None):
    """Row-major block scales [R, K/16] -> the tiled layout."""
    R, K16 = sf.shape
    return _check("metis_nvfp4_scales_to_tiled", load().metis_nvfp4_scales_to_tiled(
        _p(sf), R, K16 * 16, _p(sf_tiled), _s(stream)))


def metis_nvfp4_gemm(qa, sfa, ga, qb, sfb, gb, y, stream=None):
    """y [M, N] = NVFP4 GEMM; qa holds ceil(M/128)*128 rows, gb is a 1-element device tensor."""
    M, N = y.shape
    K = qb.shape[1] * 2
    return _check("metis_nvfp4_gemm", load().metis_nvfp4_gemm(
        _p(qa), _p(sfa), _p(ga), _p(qb), _p(sfb), _p(gb), _p(y), M, N, K, _s(stream)))


def metis_moe_nvfp4_grouped_gemm(x, topk_ids, topk_w, w_up, sf_up, g_up, w_down, sf_down, g_down,
                                 y, workspace, act=METIS_ACT_NONE, stream=None):
    """Routed-expert layer with NVFP4 experts; see the C header for shapes."""
    T, H = x.shape
    topk = topk_ids.shape[1]
    E, I, H2 = w_up.shape
    assert H2 * 2 == H
    ws_bytes = workspace.numel() * workspace.element_size()
    return _check("metis_moe_nvfp4_grouped_gemm", load().metis_moe_nvfp4_grouped_gemm(
        _p(x), _p(topk_ids), _p(topk_w), T, topk, E, H, I, _p(w_up), _p(sf_up), _p(g_up),
        _p(w_down), _p(sf_down), _p(g_down), int(act), _p(y), _p(workspace), ws_bytes,
        _s(stream)))


def metis_moe_nvfp4_workspace_offset(region, T, topk, E, H, I):
    if isinstance(region, str):
        region = MOE4_WS[region]
    return int(load().metis_moe_nvfp4_workspace_offset(int(region), int(T), int(topk), int(E),
                                                       int(H), int(I)))


# ------------------------------------------------------------ shared expert

def metis_bf16_gemm(x, w, y, stream=None):
    """y [M, N] = bf16(x [M, K] w [N, K]^T) on the tensor cores."""
    M, K = x.shape
    N = w.shape[0]
    return _check("metis_bf16_gemm", load().metis_bf16_gemm(_p(x), _p(w), _p(y), M, N, K, _s(stream)))


def metis_moe_shared_fused_combine(x, w_sup, w_sdn, o_routed, slot_to_row, topk_w, y, workspace,
                                   stream=None):
    """y = shared expert(x) + routed combine, the combine fused into the shared
    down-projection (o_routed / slot_to_row: the routed layer's workspace
    regions after it ran with y=None)."""
    T, H = x.shape
    I_s = w_sup.shape[0]
    topk = topk_w.shape[1]
    ws_bytes = workspace.numel() * workspace.element_size()
    return _check("metis_moe_shared_fused_combine", load().metis_moe_shared_fused_combine(
        _p(x), T, H, I_s, _p(w_sup), _p(w_sdn), _p(o_routed), _p(slot_to_row), _p(topk_w), topk,
        _p(y), _p(workspace), ws_bytes, _s(stream)))

