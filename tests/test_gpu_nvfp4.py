"""GPU parity of the NVFP4 path ("Lernex/Metis-1.6-Praxis-NVFP4", "What is in
NVFP4" and "What --fast-math does") against the CPU oracle, through the C ABI.

Codes, block scales and global scales are bit-exact; BF16 outputs are within
1e-2 * (1 + |ref|) of the oracle's float64 value; routing integers exact.
Each BF16 stage of the routed-expert layer is checked against the oracle on
the GPU's own input of that stage, and the layer end to end."""
import numpy as np
import pytest
import torch

import oracle
from moe_gemm_token_b200 import synth
from gpu_helpers import assert_bytes_equal, assert_close, bf16_dev, bf16_host, dev

pytestmark = pytest.mark.gpu


# --------------------------------------------------------------- layouts
# The tiled scale layout of the C header: [ceil(R/128)][K/64][512], row
# 128 a + r and block 4 c + j at byte 16 (r % 32) + 4 (r / 32) + j.

def _tiled_index(R, K):
    Rp = (R + 127) // 128 * 128
    kc = K // 64
    r = np.arange(Rp)[:, None, None]
    c = np.arange(kc)[None, :, None]
    j = np.arange(4)[None, None, :]
    off = ((r // 128) * kc + c) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + j
    return off.reshape(Rp, K // 16)


def tile_np(sf, K):
    R = sf.shape[0]
    Rp = (R + 127) // 128 * 128
    out = np.zeros(Rp * (K // 16), dtype=np.uint8)
    full = np.zeros((Rp, K // 16), dtype=np.uint8)
    full[:R] = sf
    out[_tiled_index(R, K)] = full
    return out


def untile_np(buf, rows, K):
    """Row-major scales of the given rows out of a tiled buffer."""
    idx = _tiled_index(int(np.max(rows)) + 1 if len(rows) else 1, K)
    return np.asarray(buf)[idx[np.asarray(rows)]]


def _rand_scales(rng, shape):
    s = rng.integers(0x20, 0x60, size=shape).astype(np.uint8)  # 2^-3 .. 2^5, no NaN code
    return s


# ---------------------------------------------------------- quantization

def _quant_gpu(m, x, rows_per_scale=1, tiled=False):
    R, K = x.shape
    Rp = (R + 127) // 128 * 128
    q = torch.empty((R, K // 2), dtype=torch.uint8, device="cuda")
    sf = torch.full((Rp * K // 16 if tiled else R * K // 16,), 0xAB, dtype=torch.uint8, device="cuda")
    g = torch.empty((R // rows_per_scale,), dtype=torch.float32, device="cuda")
    m.metis_quant_nvfp4(x, q, sf, g, rows_per_scale=rows_per_scale, tiled=tiled)
    torch.cuda.synchronize()
    return q.cpu().numpy(), sf.cpu().numpy(), g.cpu().numpy()


@pytest.mark.parametrize("R,K,seed", [(16, 256, 0), (37, 320, 1), (5, 2048, 2), (130, 1024, 3),
                                      (1, 64, 4), (200, 6144, 5), (3, 16384, 6)])
def test_quant_nvfp4_bf16_bit_exact(metis, R, K, seed):
    d = synth.linear(seed, R, K, 8, outlier_channels=min(4, K), outlier_scale=25.0,
                     zero_rows=(R // 2,), row_magnitude_log10=(-3, 3))
    q, sf, g = _quant_gpu(metis, bf16_dev(d["x"]))
    qr, sr, gr = oracle.nvfp4_quant(d["x"], per_row=True)
    assert_bytes_equal(g.view(np.uint32), gr.view(np.uint32), "global scales")
    assert_bytes_equal(sf.reshape(R, K // 16), sr, "block scales")
    assert_bytes_equal(oracle.e2m1_unpack(q), qr, "codes")


def test_quant_nvfp4_extremes(metis):
    """Subnormal rows (2688/amax clamped), near-BF16-max rows, signed zeros,
    E2M1 midpoints after scaling, blocks whose scale underflows to zero."""
    K = 64
    rows = [
        np.full(K, 2.0 ** -130, np.float32),
        np.linspace(-3e38, 3e38, K).astype(np.float32),
        np.where(np.arange(K) % 2 == 0, -0.0, 0.0).astype(np.float32),
        np.r_[6.0, np.tile(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0], np.float32), 8)[:K - 1]],
        np.r_[np.full(48, 1e-6, np.float32), np.full(16, 1e4, np.float32)],
        np.r_[np.full(K - 1, -1e-30, np.float32), 1.0].astype(np.float32),
    ]
    x = synth.f32_to_bf16_bits(np.stack(rows).astype(np.float32))
    q, sf, g = _quant_gpu(metis, bf16_dev(x))
    qr, sr, gr = oracle.nvfp4_quant(x, per_row=True)
    assert_bytes_equal(g.view(np.uint32), gr.view(np.uint32), "global scales")
    assert_bytes_equal(sf.reshape(x.shape[0], K // 16), sr, "block scales")
    assert_bytes_equal(oracle.e2m1_unpack(q), qr, "codes")


def test_quant_nvfp4_strided_rows(metis):
    """Rows with a leading dimension larger than K (BF16 and FP32)."""
    R, K, pad = 37, 320, 64
    d = synth.linear(9, R, K, 8, row_magnitude_log10=(-2, 2))
    qr, sr, gr = oracle.nvfp4_quant(d["x"], per_row=True)
    big = np.zeros((R, K + pad), dtype=np.uint16)
    big[:, :K] = d["x"]
    q, sf, g = _quant_gpu(metis, bf16_dev(big)[:, :K])
    assert_bytes_equal(g.view(np.uint32), gr.view(np.uint32), "global scales (BF16)")
    assert_bytes_equal(sf.reshape(R, K // 16), sr, "block scales (BF16)")
    assert_bytes_equal(oracle.e2m1_unpack(q), qr, "codes (BF16)")
    f = oracle.bf16_to_float(d["x"])
    bigf = np.zeros((R, K + pad), dtype=np.float32)
    bigf[:, :K] = f
    q, sf, g = _quant_gpu(metis, dev(bigf)[:, :K])
    assert_bytes_equal(oracle.e2m1_unpack(q), qr, "codes (FP32)")
    assert_bytes_equal(g.view(np.uint32), gr.view(np.uint32), "global scales (FP32)")


@pytest.mark.parametrize("E,N,K,seed", [(3, 128, 256, 7), (2, 384, 2048, 8)])
def test_quant_nvfp4_weight_sets_tiled(metis, E, N, K, seed):
    """FP32 expert weights [E*N, K], one global scale per expert, tiled scales."""
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((E * N, K)) * np.repeat(np.exp(rng.uniform(-3, 3, E)), N)[:, None]
         ).astype(np.float32)
    q, sf_t, g = _quant_gpu(metis, dev(w), rows_per_scale=N, tiled=True)
    q_rm, sf_rm, g_rm = _quant_gpu(metis, dev(w), rows_per_scale=N, tiled=False)
    for e in range(E):
        qr, sr, gr = oracle.nvfp4_quant(w[e * N:(e + 1) * N], per_row=False)
        assert g[e].view(np.uint32) == gr[0].view(np.uint32), f"expert {e} scale"
        assert_bytes_equal(oracle.e2m1_unpack(q[e * N:(e + 1) * N]), qr, f"expert {e} codes")
        assert_bytes_equal(sf_rm.reshape(E * N, K // 16)[e * N:(e + 1) * N], sr, f"expert {e} scales")
    assert_bytes_equal(q, q_rm, "codes independent of the scale layout")
    assert_bytes_equal(sf_t, tile_np(sf_rm.reshape(E * N, K // 16), K), "tiled layout")
    # the re-layout entry point gives the same bytes
    t2 = torch.full_like(torch.from_numpy(sf_t), 0x5A).cuda()
    metis.metis_nvfp4_scales_to_tiled(dev(sf_rm.reshape(E * N, K // 16)), t2)
    assert_bytes_equal(t2.cpu().numpy(), sf_t, "scales_to_tiled")


def test_scales_to_tiled_pads_with_zero(metis):
    rng = np.random.default_rng(3)
    R, K = 130, 192
    sf = rng.integers(0, 256, size=(R, K // 16)).astype(np.uint8)
    out = torch.full(((R + 127) // 128 * 128 * K // 16,), 0x77, dtype=torch.uint8, device="cuda")
    metis.metis_nvfp4_scales_to_tiled(dev(sf), out)
    assert_bytes_equal(out.cpu().numpy(), tile_np(sf, K), "tiled with zero pad rows")


# ------------------------------------------------------------------ GEMM

def _gemm_gpu(m, qa, sa, ga, qb, sb, gb):
    """Oracle-format operands (codes one per byte, row-major scales) -> GPU y."""
    M, K = qa.shape
    N = qb.shape[0]
    Mp = (M + 127) // 128 * 128
    qa_p = np.zeros((Mp, K // 2), dtype=np.uint8)
    qa_p[:M] = oracle.e2m1_pack(qa)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    m.metis_nvfp4_gemm(dev(qa_p), dev(tile_np(sa, K)), dev(ga), dev(oracle.e2m1_pack(qb)),
                       dev(tile_np(sb, K)), dev(np.array([gb], dtype=np.float32)), y)
    assert m.metis_check_device_status() == 0
    return bf16_host(y)


@pytest.mark.parametrize("M,N,K,seed", [(1, 128, 64, 0), (130, 256, 256, 1), (300, 384, 320, 2),
                                        (257, 512, 2048, 3), (64, 128, 4096, 4), (517, 1024, 1024, 5),
                                        (4500, 384, 256, 6)])
def test_nvfp4_gemm_parity_quantized(metis, M, N, K, seed):
    d = synth.linear(seed, M, K, N, outlier_channels=min(4, K), outlier_scale=10.0,
                     row_magnitude_log10=(-2, 2))
    qa, sa, ga = oracle.nvfp4_quant(d["x"], per_row=True)
    qb, sb, gb = oracle.nvfp4_quant(d["w"], per_row=False)
    y = _gemm_gpu(metis, qa, sa, ga, qb, sb, gb[0])
    _, y64 = oracle.nvfp4_gemm(qa, sa, ga, qb, sb, gb[0])
    assert_close(y, y64, "y")


@pytest.mark.parametrize("M,N,K,seed", [(200, 256, 512, 10), (33, 384, 192, 11)])
def test_nvfp4_gemm_parity_raw_codes(metis, M, N, K, seed):
    """Every code and a wide spread of block scales, not only quantizer output."""
    rng = np.random.default_rng(seed)
    qa = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    qb = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    sa, sb = _rand_scales(rng, (M, K // 16)), _rand_scales(rng, (N, K // 16))
    ga = rng.uniform(0.5, 2.0, M).astype(np.float32)
    y = _gemm_gpu(metis, qa, sa, ga, qb, sb, np.float32(0.375))
    _, y64 = oracle.nvfp4_gemm(qa, sa, ga, qb, sb, np.float32(0.375))
    assert_close(y, y64, "y")


def test_nvfp4_gemm_exact_small_integers(metis):
    """Unit scales and codes whose dot products are small integers: the FP32
    accumulation is exact, so y equals the oracle's rounding bit for bit."""
    rng = np.random.default_rng(12)
    M, N, K = 129, 256, 256
    qa = rng.choice([0, 2, 4, 10, 12], size=(M, K)).astype(np.uint8)  # 0, 1, 2, -1, -2
    qb = rng.choice([0, 2, 10], size=(N, K)).astype(np.uint8)
    s1 = np.full((M, K // 16), 0x38, np.uint8)
    t1 = np.full((N, K // 16), 0x38, np.uint8)
    y = _gemm_gpu(metis, qa, s1, np.ones(M, np.float32), qb, t1, np.float32(1.0))
    yr, _ = oracle.nvfp4_gemm(qa, s1, np.ones(M, np.float32), qb, t1, np.float32(1.0))
    assert_bytes_equal(y, yr, "exact y")


# --------------------------------------------------------- routed experts

def _weights_nvfp4(w):
    """[E, N, K] float32 -> (codes [E, N, K], scales [E, N, K/16], g [E]) by the oracle."""
    qs, ss, gs = [], [], []
    for e in range(w.shape[0]):
        q, s, g = oracle.nvfp4_quant(w[e], per_row=False)
        qs.append(q), ss.append(s), gs.append(g[0])
    return np.stack(qs), np.stack(ss), np.array(gs, dtype=np.float32)


def _region(m, ws, name, nbytes, T, k, E, H, I):
    off = m.metis_moe_nvfp4_workspace_offset(name, T, k, E, H, I)
    return ws[off:off + nbytes]


def run_moe4(m, d, up, dn):
    T, H, I, E, k = d["T"], d["H"], d["I"], d["E"], d["topk"]
    ws = torch.zeros((m.metis_workspace_size(m.METIS_OP_MOE_NVFP4, T, I, H, k, E),),
                     dtype=torch.uint8, device="cuda")
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    m.metis_moe_nvfp4_grouped_gemm(
        bf16_dev(d["x"]), dev(d["topk_ids"]), dev(d["topk_w"]),
        dev(oracle.e2m1_pack(up[0].reshape(E * I, H)).reshape(E, I, H // 2)),
        dev(tile_np(up[1].reshape(E * I, H // 16), H)), dev(up[2]),
        dev(oracle.e2m1_pack(dn[0].reshape(E * H, I)).reshape(E, H, I // 2)),
        dev(tile_np(dn[1].reshape(E * H, I // 16), I)), dev(dn[2]), y, ws)
    assert m.metis_check_device_status() == 0
    S = T * k
    Sp = (S + 127 * E + 127) // 128 * 128
    R = lambda name, n: _region(m, ws, name, n, T, k, E, H, I).cpu().numpy()
    return dict(
        counts=R("COUNTS", 4 * E).view(np.int32), offsets=R("OFFSETS", 4 * (E + 1)).view(np.int32),
        s2r=R("SLOT_TO_ROW", 4 * S).view(np.int32), r2s=R("ROW_TO_SLOT", 4 * Sp).view(np.int32),
        aq=R("AQ", Sp * H // 2).reshape(Sp, H // 2), sfa=R("SFA", Sp * H // 16),
        ga=R("GA", 4 * Sp).view(np.float32),
        h=R("H", 2 * Sp * I).view(np.uint16).reshape(Sp, I), hq=R("HQ", Sp * I // 2).reshape(Sp, I // 2),
        sfh=R("SFH", Sp * I // 16), gh=R("GH", 4 * Sp).view(np.float32),
        o=R("O", 2 * Sp * H).view(np.uint16).reshape(Sp, H), y=bf16_host(y))


def check_moe4(d, g, up, dn, tokens=None):
    T, k, E, H, I = d["T"], d["topk"], d["E"], d["H"], d["I"]
    ids = d["topk_ids"]
    counts, offsets, s2r, _ = oracle.moe_route(ids, E)
    padded = np.r_[0, np.cumsum((counts + 127) // 128 * 128)].astype(np.int32)
    exp_all = ids.reshape(-1)
    rows_all = padded[exp_all] + (s2r - offsets[exp_all])
    assert_bytes_equal(g["counts"], counts, "counts")
    assert_bytes_equal(g["offsets"], padded, "padded offsets")
    assert_bytes_equal(g["s2r"], rows_all, "slot_to_row")
    assert_bytes_equal(g["r2s"][rows_all], np.arange(T * k, dtype=np.int32), "row_to_slot")
    pad = np.ones(padded[-1], bool)
    pad[rows_all] = False
    assert np.all(g["r2s"][:padded[-1]][pad] == -1), "pad rows marked"
    # x in NVFP4, written into every row its token was routed to
    qx, sx, gx = oracle.nvfp4_quant(d["x"], per_row=True)
    tok_all = np.arange(T * k) // k
    assert_bytes_equal(oracle.e2m1_unpack(g["aq"][rows_all]), qx[tok_all], "x codes in expert order")
    assert_bytes_equal(untile_np(g["sfa"], rows_all, H), sx[tok_all], "x block scales in expert order")
    assert_bytes_equal(g["ga"][rows_all].view(np.uint32), gx[tok_all].view(np.uint32), "x global scales")
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    slots = (toks[:, None] * k + np.arange(k)).reshape(-1)
    rows, exp, tok = rows_all[slots], exp_all[slots], tok_all[slots]
    # up-projection on the GPU's operands
    h64 = np.empty((slots.size, I))
    for e in np.unique(exp):
        sel = np.nonzero(exp == e)[0]
        _, h64[sel] = oracle.nvfp4_gemm(qx[tok[sel]], sx[tok[sel]], gx[tok[sel]], up[0][e], up[1][e],
                                        up[2][e])
    assert_close(g["h"][rows], h64, "h")
    # re-quantization of the GPU's h: bit-exact
    qh, sh, gh = oracle.nvfp4_quant(g["h"][rows], per_row=True)
    assert_bytes_equal(oracle.e2m1_unpack(g["hq"][rows]), qh, "h codes")
    assert_bytes_equal(untile_np(g["sfh"], rows, I), sh, "h block scales")
    assert_bytes_equal(g["gh"][rows].view(np.uint32), gh.view(np.uint32), "h global scales")
    # down-projection on the GPU's codes
    o64 = np.empty((slots.size, H))
    for e in np.unique(exp):
        sel = np.nonzero(exp == e)[0]
        _, o64[sel] = oracle.nvfp4_gemm(qh[sel], sh[sel], gh[sel], dn[0][e], dn[1][e], dn[2][e])
    assert_close(g["o"][rows], o64, "o")
    # combine on the GPU's o, then the whole layer against the oracle alone
    _, y64 = oracle.moe_combine(g["o"][rows].reshape(toks.size, k, H), d["topk_w"][toks])
    assert_close(g["y"][toks], y64, "y (combine)")
    ref = oracle.moe_forward_nvfp4(d["x"], ids, d["topk_w"], up, dn, tokens=toks)
    assert_close(g["y"][toks], ref["y64"], "y (end to end)")


@pytest.mark.parametrize("T,H,I,E,k,seed", [(200, 256, 128, 8, 2, 11), (300, 512, 256, 64, 8, 12),
                                            (37, 128, 384, 5, 3, 13), (1, 128, 128, 4, 4, 14),
                                            (513, 256, 512, 16, 1, 15), (96, 2048, 256, 16, 4, 18)])
def test_moe_nvfp4_parity(metis, T, H, I, E, k, seed):
    d = synth.moe(seed=seed, T=T, H=H, I=I, E=E, topk=k, hot=min(2, E), load_ratio=2.0)
    up, dn = _weights_nvfp4(d["w_up"]), _weights_nvfp4(d["w_down"])
    g = run_moe4(metis, d, up, dn)
    check_moe4(d, g, up, dn)


@pytest.mark.parametrize("E,seed", [(256, 19), (320, 20)])
def test_moe_nvfp4_many_experts(metis, E, seed):
    """256 experts (group tables and pad marking at larger E; the fused
    prefix-sum and rank kernel) and 320 (past its 256-expert limit: the
    single-block scan, which marks the pad rows, then the rank kernel), top-4."""
    d = synth.moe(seed=seed, T=96, H=128, I=128, E=E, topk=4, hot=4, load_ratio=2.0)
    up, dn = _weights_nvfp4(d["w_up"]), _weights_nvfp4(d["w_down"])
    g = run_moe4(metis, d, up, dn)
    check_moe4(d, g, up, dn)


def test_moe_nvfp4_empty_experts_and_determinism(metis):
    d = synth.moe(seed=16, T=64, H=128, I=128, E=16, topk=2, hot=0, load_ratio=1.0)
    ids = d["topk_ids"]
    ids[ids >= 12] = ids[ids >= 12] % 4     # experts 12..15 get nothing
    for t in range(ids.shape[0]):           # keep each token's experts distinct
        if ids[t, 0] == ids[t, 1]:
            ids[t, 1] = (ids[t, 0] + 1) % 12
    d["topk_ids"] = ids
    up, dn = _weights_nvfp4(d["w_up"]), _weights_nvfp4(d["w_down"])
    g1 = run_moe4(metis, d, up, dn)
    check_moe4(d, g1, up, dn)
    g2 = run_moe4(metis, d, up, dn)
    assert_bytes_equal(g1["y"], g2["y"], "run-to-run")


def test_moe_nvfp4_full_size(metis):
    """The workload the bench times (4096 tokens, hidden 2048, latent 1024,
    64 experts, top-8, four hot experts), checked on sampled tokens."""
    d = synth.moe()
    up, dn = _weights_nvfp4(d["w_up"]), _weights_nvfp4(d["w_down"])
    g = run_moe4(metis, d, up, dn)
    ids = d["topk_ids"]
    rng = np.random.default_rng(1)
    hot_tok = np.nonzero(np.isin(ids, d["hot_experts"]).any(axis=1))[0]
    toks = np.unique(np.r_[rng.choice(d["T"], 24, replace=False), hot_tok[:8], 0, d["T"] - 1])
    check_moe4(d, g, up, dn, tokens=toks)


@pytest.mark.parametrize("M,N,K", [(8192, 4096, 4096)])
def test_nvfp4_gemm_full_size_sampled(metis, M, N, K):
    """The dense NVFP4 GEMM at a bench size, quantized on the GPU, sampled rows."""
    d = synth.large_m(M=M, K=K)
    x = bf16_dev(d["x"])
    Mp = (M + 127) // 128 * 128
    qa = torch.empty((Mp, K // 2), dtype=torch.uint8, device="cuda")
    sa = torch.empty((Mp * K // 16,), dtype=torch.uint8, device="cuda")
    ga = torch.empty((M,), dtype=torch.float32, device="cuda")
    metis.metis_quant_nvfp4(x, qa[:M], sa, ga, tiled=True)
    w = dev(d["w"][:N])
    qb = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    sb = torch.empty((N * K // 16,), dtype=torch.uint8, device="cuda")
    gb = torch.empty((1,), dtype=torch.float32, device="cuda")
    metis.metis_quant_nvfp4(w, qb, sb, gb, rows_per_scale=N, tiled=True)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_nvfp4_gemm(qa, sa, ga, qb, sb, gb, y)
    assert metis.metis_check_device_status() == 0
    rows = np.unique(np.r_[np.random.default_rng(2).choice(M, 30, replace=False), 0, M - 1])
    qa_r, sa_r, ga_r = oracle.nvfp4_quant(d["x"][rows], per_row=True)
    qb_r, sb_r, gb_r = oracle.nvfp4_quant(d["w"][:N], per_row=False)
    assert_bytes_equal(oracle.e2m1_unpack(qa.cpu().numpy()[rows]), qa_r, "A codes")
    assert_bytes_equal(untile_np(sa.cpu().numpy(), rows, K), sa_r, "A scales")
    assert_bytes_equal(gb.cpu().numpy().view(np.uint32), gb_r.view(np.uint32), "B global scale")
    _, y64 = oracle.nvfp4_gemm(qa_r, sa_r, ga_r, qb_r, sb_r, gb_r[0])
    assert_close(bf16_host(y)[rows], y64, "y")

