"""CPU oracle for the FP8 fast-math linear layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
(and its ``--impl reference`` arm) may import this package. The product path
(``moe_gemm_token_b200``) never imports it and shares no code with it.

The arithmetic lives in ``metis_oracle.c`` (plain loops, float64 sums, one
rounding at the end); this module only marshals numpy arrays into it and
composes its steps for the routed-expert path in the order the model cards
describe them:

* "Lernex/Metis-1.6-Logos-FP8" model card, "What --fast-math does": each
  layer's input rounded to FP8 per token, then multiplied with the FP8
  weights; the default widens the FP8 weights and does BF16 maths.
* same card, "What is in FP8": E4M3 weights with one scale per output channel,
  activations quantized per token at run time; routed experts are FP8.

BF16 tensors are carried as ``uint16`` bit patterns throughout.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.metis_oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.metis_oracle_e4m3_decode.restype = ctypes.c_double
        lib.metis_oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.metis_oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.metis_oracle_bf16_from_double.argtypes = [ctypes.c_double]
        lib.metis_oracle_bf16_from_double.restype = ctypes.c_uint16
        lib.metis_oracle_quant_rows_bf16.argtypes = [p, i64, i64, i64, p, i64, p]
        lib.metis_oracle_quant_rows_f32.argtypes = [p, i64, i64, i64, p, i64, p]
        lib.metis_oracle_gemm_w8a8.argtypes = [p, i64, p, p, i64, p, i64, i64, i64, p, i64, p, p]
        lib.metis_oracle_gemm_w8a16.argtypes = [p, i64, p, i64, p, i64, i64, i64, p, p]
        lib.metis_oracle_moe_route.argtypes = [p, i64, i64, i64, p, p, p, p]
        lib.metis_oracle_moe_combine.argtypes = [p, p, i64, i64, i64, p, p]
        lib.metis_oracle_e4m3_encode_array.argtypes = [p, i64, p]
        lib.metis_oracle_e4m3_decode_array.argtypes = [p, i64, p]
        lib.metis_oracle_bf16_from_double_array.argtypes = [p, i64, p]
        lib.metis_oracle_route_topk.argtypes = [p, p, i64, i64, i64, p, p]
        lib.metis_oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.metis_oracle_e2m1_decode.restype = ctypes.c_double
        lib.metis_oracle_e2m1_encode.argtypes = [ctypes.c_float]
        lib.metis_oracle_e2m1_encode.restype = ctypes.c_uint8
        lib.metis_oracle_nvfp4_quant.argtypes = [p, i64, i64, ctypes.c_int, p, p, p]
        lib.metis_oracle_nvfp4_gemm.argtypes = [p, p, p, p, p, ctypes.c_float, i64, i64, i64, p, p]
        lib.metis_oracle_gemm_bf16.argtypes = [p, i64, p, i64, i64, i64, i64, p, p]
        lib.metis_oracle_shared_combine.argtypes = [p, p, p, i64, i64, i64, p, p]
        for name in ("route_topk", "nvfp4_quant", "nvfp4_gemm", "gemm_bf16", "shared_combine"):
            getattr(lib, "metis_oracle_" + name).restype = ctypes.c_int
        for name in ("e4m3_encode_array", "e4m3_decode_array", "bf16_from_double_array"):
            getattr(lib, "metis_oracle_" + name).restype = None
        for name in ("quant_rows_bf16", "quant_rows_f32", "gemm_w8a8", "gemm_w8a16",
                     "moe_route", "moe_combine"):
            getattr(lib, "metis_oracle_" + name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


# ------------------------------------------------------------------ codec

def e4m3_decode(b):
    """Exact value of each E4M3 byte (OCP OFP8 E4M3), as float64."""
    lib = _load()
    b = _c(b, np.uint8)
    out = np.empty(b.shape, dtype=np.float64)
    lib.metis_oracle_e4m3_decode_array(_ptr(b), b.size, _ptr(out))
    return out


def e4m3_decode_table():
    """The 256-entry decode table D(b), b = 0..255."""
    return e4m3_decode(np.arange(256, dtype=np.uint8))


def e4m3_encode(v):
    """Q(v): binary32 -> E4M3 byte, nearest-even, saturating to +-448."""
    lib = _load()
    v = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib.metis_oracle_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def bf16_from_double(v):
    """Round float64 values once to BF16 (nearest-even); returns uint16 bits."""
    lib = _load()
    v = _c(v, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib.metis_oracle_bf16_from_double_array(_ptr(v), v.size, _ptr(out))
    return out


def bf16_to_float(h):
    """Exact widening of BF16 bit patterns to float32."""
    h = np.asarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------- quantization

def quant_per_token(x_bf16):
    """Per-token FP8 quantization of BF16 activations [M, K].

    Returns (codes uint8 [M, K], scales float32 [M]) with s = amax/448 and
    codes Q(x * 448/amax)."""
    lib = _load()
    x = _c(x_bf16, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((M,), dtype=np.float32)
    _check(lib.metis_oracle_quant_rows_bf16(_ptr(x), M, K, K, _ptr(q), K, _ptr(s)),
           "quant_rows_bf16")
    return q, s


def quant_per_channel(w_f32):
    """Per-output-channel FP8 quantization of float32 weights [N, K]."""
    lib = _load()
    w = _c(w_f32, np.float32)
    N, K = w.shape
    q = np.empty((N, K), dtype=np.uint8)
    s = np.empty((N,), dtype=np.float32)
    _check(lib.metis_oracle_quant_rows_f32(_ptr(w), N, K, K, _ptr(q), K, _ptr(s)),
           "quant_rows_f32")
    return q, s


# ------------------------------------------------------------------ GEMMs

def gemm_w8a8(xq, s_tok, wq, s_w, rows=None):
    """W8A8 fast-math GEMM: bf16(s_tok[m] s_w[n] sum_k D(xq[m,k]) D(wq[n,k])).

    ``rows`` selects output rows (default: all). Returns (bf16 bits [R, N],
    float64 values before the final rounding [R, N])."""
    lib = _load()
    xq = _c(xq, np.uint8)
    wq = _c(wq, np.uint8)
    s_tok = _c(s_tok, np.float32)
    s_w = _c(s_w, np.float32)
    M, K = xq.shape
    N, K2 = wq.shape
    assert K == K2
    if rows is None:
        r = None
        R = M
    else:
        r = _c(rows, np.int64)
        R = r.size
    y = np.empty((R, N), dtype=np.uint16)
    y64 = np.empty((R, N), dtype=np.float64)
    _check(lib.metis_oracle_gemm_w8a8(_ptr(xq), K, _ptr(s_tok), _ptr(wq), K, _ptr(s_w),
                                      M, N, K, _ptr(r), R, _ptr(y), _ptr(y64)), "gemm_w8a8")
    return y, y64


def gemm_w8a16(x_bf16, wq, s_w):
    """W8A16 default maths: bf16(s_w[n] sum_k x[m,k] D(wq[n,k])), float64 sum."""
    lib = _load()
    x = _c(x_bf16, np.uint16)
    wq = _c(wq, np.uint8)
    s_w = _c(s_w, np.float32)
    M, K = x.shape
    N, K2 = wq.shape
    assert K == K2
    y = np.empty((M, N), dtype=np.uint16)
    y64 = np.empty((M, N), dtype=np.float64)
    _check(lib.metis_oracle_gemm_w8a16(_ptr(x), K, _ptr(wq), K, _ptr(s_w), M, N, K,
                                       _ptr(y), _ptr(y64)), "gemm_w8a16")
    return y, y64


def linear_w8a8(x_bf16, wq, s_w, rows=None):
    """The fast-math linear layer end to end: per-token quantization of the
    BF16 input, then the W8A8 GEMM. Returns (y bf16 bits, y float64, xq, s_tok)."""
    xq, s_tok = quant_per_token(x_bf16)
    y, y64 = gemm_w8a8(xq, s_tok, wq, s_w, rows=rows)
    return y, y64, xq, s_tok


# --------------------------------------------------------- routed experts

def moe_route(topk_ids, num_experts):
    """Histogram, exclusive prefix sum and stable permutation of the routed
    slots s = t*topk + j. Returns (counts [E], offsets [E+1],
    slot_to_row [T*k], row_to_slot [T*k]) as int32."""
    lib = _load()
    ids = _c(topk_ids, np.int32)
    T, k = ids.shape
    E = int(num_experts)
    counts = np.empty((E,), dtype=np.int32)
    offsets = np.empty((E + 1,), dtype=np.int32)
    s2r = np.empty((T * k,), dtype=np.int32)
    r2s = np.empty((T * k,), dtype=np.int32)
    _check(lib.metis_oracle_moe_route(_ptr(ids), T, k, E, _ptr(counts), _ptr(offsets),
                                      _ptr(s2r), _ptr(r2s)), "moe_route")
    # counts were reused as fill cursors and end equal to the histogram again
    return counts, offsets, s2r, r2s


def route_topk(logits, topk, bias=None):
    """Router top-k on binary32 logits [T, E] (+ optional binary32 balance bias
    [E] that only decides the choice): ids [T, k] int32 in descending score
    order (ties to the lower expert), weights [T, k] float64, a softmax over
    the chosen experts' own logits."""
    lib = _load()
    lg = _c(logits, np.float32)
    T, E = lg.shape
    b = None if bias is None else _c(bias, np.float32)
    ids = np.empty((T, topk), dtype=np.int32)
    w = np.empty((T, topk), dtype=np.float64)
    _check(lib.metis_oracle_route_topk(_ptr(lg), _ptr(b), T, E, int(topk), _ptr(ids), _ptr(w)),
           "route_topk")
    return ids, w


def moe_combine(o_slots_bf16, topk_w):
    """y[t] = bf16(sum_j w[t,j] o[t,j]) with o in slot order [T, k, H] (bf16 bits)."""
    lib = _load()
    o = _c(o_slots_bf16, np.uint16)
    w = _c(topk_w, np.float32)
    T, k, H = o.shape
    y = np.empty((T, H), dtype=np.uint16)
    y64 = np.empty((T, H), dtype=np.float64)
    _check(lib.metis_oracle_moe_combine(_ptr(o), _ptr(w), T, k, H, _ptr(y), _ptr(y64)),
           "moe_combine")
    return y, y64


def moe_expert_gemm(aq, s_a, wq_experts, s_w_experts, slot_expert, slots=None):
    """Per-slot W8A8 GEMM against the slot's own expert.

    ``aq``/``s_a`` hold one quantized row operand per slot and
    ``slot_expert[s]`` names the slot's expert. Returns (bf16 bits [S, N],
    float64 [S, N]) for the chosen slots (default: all rows of ``aq``)."""
    S_all = aq.shape[0]
    slots = np.arange(S_all) if slots is None else np.asarray(slots, dtype=np.int64)
    N = wq_experts.shape[1]
    y = np.empty((slots.size, N), dtype=np.uint16)
    y64 = np.empty((slots.size, N), dtype=np.float64)
    experts = np.asarray(slot_expert)[slots]
    for e in np.unique(experts):
        sel = np.nonzero(experts == e)[0]
        ye, y64e = gemm_w8a8(aq, s_a, wq_experts[e], s_w_experts[e], rows=slots[sel])
        y[sel] = ye
        y64[sel] = y64e
    return y, y64


def moe_forward(x_bf16, topk_ids, topk_w, w_up, s_up, w_down, s_down, tokens=None):
    """Routed-expert W8A8 layer for the chosen tokens (default: all).

    Steps, in the order the fast-math description implies for each FP8
    projection: quantize x per token; per routed slot (t, j) with expert
    e = ids[t, j], up-projection h = bf16(s_x[t] s_up[e,n] sum D(xq) D(w_up[e]));
    no activation between the projections; quantize h per row; down-projection
    o = bf16(s_h s_down[e,n] sum D(hq) D(w_down[e])); combine
    y[t] = bf16(sum_j w[t,j] o[t,j]) in float64.

    Returns a dict with every intermediate (rows ordered by selected token,
    then j)."""
    x = _c(x_bf16, np.uint16)
    ids = _c(topk_ids, np.int32)
    w = _c(topk_w, np.float32)
    T, k = ids.shape
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    xq, s_x = quant_per_token(x[tokens])
    nt = tokens.size
    # one row operand per (selected token, j)
    slot_tok = np.repeat(np.arange(nt), k)
    slot_exp = ids[tokens].reshape(-1)
    aq = xq[slot_tok]
    s_a = s_x[slot_tok]
    h, h64 = moe_expert_gemm(aq, s_a, w_up, s_up, slot_exp)
    hq, s_h = quant_per_token(h)
    o, o64 = moe_expert_gemm(hq, s_h, w_down, s_down, slot_exp)
    y, y64 = moe_combine(o.reshape(nt, k, -1), w[tokens])
    return dict(xq=xq, s_x=s_x, h=h, h64=h64, hq=hq, s_h=s_h, o=o, o64=o64, y=y, y64=y64,
                tokens=tokens)


# ------------------------------------------------------------------ NVFP4
# "Lernex/Metis-1.6-Praxis-NVFP4", "What is in NVFP4": routed experts hold
# 4-bit E2M1 values, one E4M3 scale per 16 inputs and one FP32 scale per
# expert; "What --fast-math does": with fast-math their inputs are rounded to
# FP4 as well. The scale rule (global scale amax/2688 = amax/(6 * 448), block
# scale E4M3(block amax * (2688/amax) / 6)) is this oracle's reading; the
# pages print none. Codes are carried one per byte here; the library's packed
# form (two codes per byte, the even k in the low nibble) is converted by
# e2m1_pack / e2m1_unpack, which do no arithmetic.

def e2m1_decode(c):
    """Exact value of each E2M1 code (low 4 bits), as float64."""
    lib = _load()
    c = np.asarray(c, dtype=np.uint8)
    return np.vectorize(lambda b: lib.metis_oracle_e2m1_decode(int(b)), otypes=[np.float64])(c) \
        if c.size else np.zeros(c.shape)


def e2m1_encode(v):
    """binary32 -> E2M1 code: nearest of +-{0, .5, 1, 1.5, 2, 3, 4, 6}, ties to
    the even mantissa, saturating to +-6."""
    lib = _load()
    v = _c(v, np.float32)
    return np.vectorize(lambda x: lib.metis_oracle_e2m1_encode(float(x)), otypes=[np.uint8])(v) \
        if v.size else np.zeros(v.shape, dtype=np.uint8)


def e2m1_pack(q):
    """[R, K] codes (one per byte) -> [R, K/2] bytes, code of k = 2i in the low nibble."""
    q = np.asarray(q, dtype=np.uint8)
    return (q[..., 0::2] & 0xF) | ((q[..., 1::2] & 0xF) << 4)


def e2m1_unpack(b):
    """[R, K/2] packed bytes -> [R, K] codes."""
    b = np.asarray(b, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def nvfp4_quant(x, per_row=True):
    """NVFP4 quantization of rows [R, K] (K % 16 == 0) given as float32, or as
    BF16 bit patterns (uint16, widened exactly).

    per_row: one global scale per row (activations, per token); otherwise one
    for the whole matrix (an expert's weights). Returns (codes uint8 [R, K],
    block scales uint8 E4M3 codes [R, K/16], g float32 [R] or [1])."""
    lib = _load()
    x = np.asarray(x)
    if x.dtype == np.uint16:
        x = bf16_to_float(x)
    x = _c(x, np.float32)
    R, K = x.shape
    q = np.empty((R, K), dtype=np.uint8)
    sb = np.empty((R, K // 16), dtype=np.uint8)
    g = np.empty((R if per_row else 1,), dtype=np.float32)
    _check(lib.metis_oracle_nvfp4_quant(_ptr(x), R, K, int(bool(per_row)), _ptr(q), _ptr(sb),
                                        _ptr(g)), "nvfp4_quant")
    return q, sb, g


def nvfp4_dequant(q, sb, g):
    """D2(q) * D(sb) * g as float64 ([R, K]); g has one entry per row or one."""
    q = np.asarray(q, dtype=np.uint8)
    R, K = q.shape
    v = e2m1_decode(q) * np.repeat(e4m3_decode(sb), 16, axis=1)
    g = np.asarray(g, dtype=np.float64)
    return v * (g.reshape(-1, 1) if g.size == R else g.reshape(1, 1))


def nvfp4_gemm(qa, sa, ga, qb, sbb, gb, rows=None):
    """y[m, n] = bf16(ga[m] gb sum_k D2(qa) D(sa) D2(qb) D(sbb)), float64 sum.

    qa [M, K] codes, sa [M, K/16], ga [M]; qb [N, K], sbb [N, K/16], gb one
    float. ``rows`` selects rows of A (default all). Returns (bf16 bits,
    float64 before rounding)."""
    lib = _load()
    if rows is not None:
        rows = np.asarray(rows, dtype=np.int64)
        qa, sa, ga = np.asarray(qa)[rows], np.asarray(sa)[rows], np.asarray(ga)[rows]
    qa, sa, ga = _c(qa, np.uint8), _c(sa, np.uint8), _c(ga, np.float32)
    qb, sbb = _c(qb, np.uint8), _c(sbb, np.uint8)
    M, K = qa.shape
    N = qb.shape[0]
    y = np.empty((M, N), dtype=np.uint16)
    y64 = np.empty((M, N), dtype=np.float64)
    _check(lib.metis_oracle_nvfp4_gemm(_ptr(qa), _ptr(sa), _ptr(ga), _ptr(qb), _ptr(sbb),
                                       float(np.float32(gb)), M, N, K, _ptr(y), _ptr(y64)),
           "nvfp4_gemm")
    return y, y64


def moe_forward_nvfp4(x_bf16, topk_ids, topk_w, up, down, tokens=None):
    """Routed-expert layer with NVFP4 experts under fast-math.

    ``up`` / ``down`` are (codes [E, N, K], block scales [E, N, K/16], g [E])
    per projection. Steps: x quantized to NVFP4 per token; per routed slot
    (t, j), e = ids[t, j]: h = bf16(g_x[t] g_up[e] sum ...); h quantized to
    NVFP4 per slot row; o = bf16(g_h g_dn[e] sum ...); y[t] = bf16(sum_j
    w[t, j] o[t, j]) in float64. Returns every intermediate, rows ordered by
    selected token, then j."""
    x = _c(x_bf16, np.uint16)
    ids = _c(topk_ids, np.int32)
    w = _c(topk_w, np.float32)
    T, k = ids.shape
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    qx, sx, gx = nvfp4_quant(x[tokens], per_row=True)
    nt = tokens.size
    slot_tok = np.repeat(np.arange(nt), k)
    slot_exp = ids[tokens].reshape(-1)

    def expert_gemm(qa, sa, ga, wts):
        qw, sw, gw = wts
        N = qw.shape[1]
        y = np.empty((qa.shape[0], N), dtype=np.uint16)
        y64 = np.empty((qa.shape[0], N), dtype=np.float64)
        for e in np.unique(slot_exp):
            sel = np.nonzero(slot_exp == e)[0]
            ye, y64e = nvfp4_gemm(qa[sel], sa[sel], ga[sel], qw[e], sw[e], gw[e])
            y[sel] = ye
            y64[sel] = y64e
        return y, y64

    h, h64 = expert_gemm(qx[slot_tok], sx[slot_tok], gx[slot_tok], up)
    qh, sh, gh = nvfp4_quant(h, per_row=True)
    o, o64 = expert_gemm(qh, sh, gh, down)
    y, y64 = moe_combine(o.reshape(nt, k, -1), w[tokens])
    return dict(qx=qx, sx=sx, gx=gx, h=h, h64=h64, qh=qh, sh=sh, gh=gh, o=o, o64=o64, y=y,
                y64=y64, tokens=tokens)


# ------------------------------------------------------------ shared expert
# "Lernex/Metis-1.6-Praxis" card, "Architecture": one shared expert beside
# the routed ones in every layer; the FP8 cards ("What is in FP8") keep it in
# BF16. Reading: it runs on every token with weight 1, with the two
# projections of a routed expert (no activation, h rounded to BF16), and its
# BF16 output joins the routed weighted sum before the final rounding.

def gemm_bf16(x_bf16, w_bf16, rows=None):
    """y[m, n] = bf16(sum_k x[m, k] w[n, k]) with BF16 operands, float64 sum.
    Returns (bf16 bits, float64 before rounding)."""
    lib = _load()
    x = _c(x_bf16, np.uint16)
    if rows is not None:
        x = np.ascontiguousarray(x[np.asarray(rows)])
    w = _c(w_bf16, np.uint16)
    M, K = x.shape
    N = w.shape[0]
    y = np.empty((M, N), dtype=np.uint16)
    y64 = np.empty((M, N), dtype=np.float64)
    _check(lib.metis_oracle_gemm_bf16(_ptr(x), K, _ptr(w), K, M, N, K, _ptr(y), _ptr(y64)),
           "gemm_bf16")
    return y, y64


def shared_combine(s_bf16, o_slots_bf16, topk_w):
    """y[t] = bf16(s[t] + sum_j w[t, j] o[t, j]) in float64; s [T, H], o [T, k, H]."""
    lib = _load()
    s = _c(s_bf16, np.uint16)
    o = _c(o_slots_bf16, np.uint16)
    w = _c(topk_w, np.float32)
    T, k, H = o.shape
    y = np.empty((T, H), dtype=np.uint16)
    y64 = np.empty((T, H), dtype=np.float64)
    _check(lib.metis_oracle_shared_combine(_ptr(s), _ptr(o), _ptr(w), T, k, H, _ptr(y), _ptr(y64)),
           "shared_combine")
    return y, y64


def shared_expert(x_bf16, w_sup_bf16, w_sdn_bf16, tokens=None):
    """The shared expert's BF16 output: s = bf16(bf16(x W_up^T) W_down^T).
    Returns (h bits, s bits, s float64)."""
    h, _ = gemm_bf16(x_bf16, w_sup_bf16, rows=tokens)
    s, s64 = gemm_bf16(h, w_sdn_bf16)
    return h, s, s64

