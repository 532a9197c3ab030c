"""GPU parity of the BF16 GEMM and of the shared expert joined to the routed
combine ("Lernex/Metis-1.6-Praxis" card, "Architecture": one shared expert
beside the routed ones; the FP8 cards keep it in BF16), against the CPU oracle
through the C ABI. BF16 outputs within 1e-2 * (1 + |ref|); the combine with a
zero shared expert is bit-exact with the routed layer's own combine kernel."""
import numpy as np
import pytest
import torch

import oracle
from moe_gemm_token_b200 import synth
from gpu_helpers import assert_bytes_equal, assert_close, bf16_dev, bf16_host, dev
from test_gpu_moe import run_moe
from test_gpu_nvfp4 import _weights_nvfp4, run_moe4

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K,seed", [(1, 8, 8, 0), (130, 256, 256, 1), (300, 384, 328, 2),
                                        (512, 1024, 2048, 3), (77, 136, 1000, 4), (4500, 264, 128, 5)])
def test_bf16_gemm_parity(metis, M, N, K, seed):
    rng = np.random.default_rng(seed)
    x = synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    w = synth.f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.05).astype(np.float32))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_bf16_gemm(bf16_dev(x), bf16_dev(w), y)
    assert metis.metis_check_device_status() == 0
    _, y64 = oracle.gemm_bf16(x, w)
    assert_close(bf16_host(y), y64, "y")


def _shared_weights(seed, H, I_s, scale=0.03):
    rng = np.random.default_rng(seed)
    wu = synth.f32_to_bf16_bits((rng.standard_normal((I_s, H)) * scale).astype(np.float32))
    wd = synth.f32_to_bf16_bits((rng.standard_normal((H, I_s)) * scale).astype(np.float32))
    return wu, wd


def _region(ws, off, n, dtype):
    return ws[off:off + n * torch.empty((), dtype=dtype).element_size()].view(dtype)


def _run_fused(metis, d, wu, wd, o_dev, s2r_dev):
    T, H = d["x"].shape
    I_s = wu.shape[0]
    k = d["topk"]
    ws = torch.zeros((metis.metis_workspace_size(metis.METIS_OP_SHARED, T, I_s, H, k, 0),),
                     dtype=torch.uint8, device="cuda")
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    metis.metis_moe_shared_fused_combine(bf16_dev(d["x"]), bf16_dev(wu), bf16_dev(wd), o_dev, s2r_dev,
                                         dev(d["topk_w"]), y, ws)
    assert metis.metis_check_device_status() == 0
    hs = ws[:2 * T * I_s].view(torch.int16).view(T, I_s).cpu().numpy().view(np.uint16)
    s_off = (2 * T * I_s + 255) // 256 * 256   # the shared output s [T, H] follows h_s
    s = ws[s_off:s_off + 2 * T * H].view(torch.int16).view(T, H).cpu().numpy().view(np.uint16)
    _, s64 = oracle.gemm_bf16(hs, wd)   # s is the GPU's h_s through the down-projection
    assert_close(s, s64, "shared output s")
    return bf16_host(y), hs


def _check_fused(d, wu, wd, y, hs, o_rows, tokens=None):
    """o_rows: the GPU's routed outputs in slot order [T, k, H] (bf16 bits)."""
    toks = np.arange(d["x"].shape[0]) if tokens is None else np.asarray(tokens)
    _, hs64 = oracle.gemm_bf16(d["x"], wu, rows=toks)
    assert_close(hs[toks], hs64, "shared h")
    s, _ = oracle.gemm_bf16(hs[toks], wd)           # the shared output on the GPU's h_s
    _, y64 = oracle.shared_combine(s, o_rows[toks], d["topk_w"][toks])
    assert_close(y[toks], y64, "y")
    # end to end: the oracle's own shared expert and the same routed outputs
    _, s_ref, _ = oracle.shared_expert(d["x"], wu, wd, tokens=toks)
    _, y64r = oracle.shared_combine(s_ref, o_rows[toks], d["topk_w"][toks])
    assert_close(y[toks], y64r, "y (oracle shared expert)")


def _o_slots(g, rows, T, k):
    return g["o"][rows].reshape(T, k, -1)


@pytest.mark.parametrize("T,H,I,I_s,E,k,seed", [(200, 256, 128, 256, 8, 2, 21), (300, 512, 256, 128, 64, 8, 22),
                                                (37, 128, 272, 64, 5, 3, 23)])
def test_shared_fused_combine_fp8_routed(metis, T, H, I, I_s, E, k, seed):
    d = synth.moe(seed=seed, T=T, H=H, I=I, E=E, topk=k, hot=min(2, E), load_ratio=2.0)
    g = run_moe(metis, d)   # routed layer with its own combine (for the zero-shared check)
    S = T * k
    ws_off = lambda name: metis.metis_moe_workspace_offset(name, T, k, E, H, I)
    # the routed outputs and slot->row map, as the routed layer left them
    o_dev = dev(g["o"].view(np.int16)).view(torch.bfloat16)
    s2r_dev = dev(g["s2r"])
    wu, wd = _shared_weights(seed, H, I_s)
    y, hs = _run_fused(metis, d, wu, wd, o_dev, s2r_dev)
    _check_fused(d, wu, wd, y, hs, _o_slots(g, g["s2r"], T, k))
    # a zero shared expert: the fused combine is the routed combine, bit for bit
    z = np.zeros_like(wu), np.zeros_like(wd)
    y0, _ = _run_fused(metis, d, z[0], z[1], o_dev, s2r_dev)
    assert_bytes_equal(y0, g["y"], "zero shared expert = routed combine")
    assert ws_off("O") >= 0 and S > 0


def test_shared_fused_combine_nvfp4_routed_and_null_y(metis):
    """The NVFP4 routed layer with y = NULL leaves o in the workspace; the fused
    shared combine finishes the layer."""
    T, H, I, I_s, E, k = 160, 256, 256, 128, 16, 4
    d = synth.moe(seed=24, T=T, H=H, I=I, E=E, topk=k, hot=2, load_ratio=2.0)
    up, dn = _weights_nvfp4(d["w_up"]), _weights_nvfp4(d["w_down"])
    g = run_moe4(metis, d, up, dn)   # with y: reference routed combine
    # again with y = NULL into a fresh workspace
    ws = torch.zeros((metis.metis_workspace_size(metis.METIS_OP_MOE_NVFP4, T, I, H, k, E),),
                     dtype=torch.uint8, device="cuda")
    metis.metis_moe_nvfp4_grouped_gemm(
        bf16_dev(d["x"]), dev(d["topk_ids"]), dev(d["topk_w"]),
        dev(oracle.e2m1_pack(up[0].reshape(E * I, H)).reshape(E, I, H // 2)),
        dev(_tile(up[1].reshape(E * I, H // 16), H)), dev(up[2]),
        dev(oracle.e2m1_pack(dn[0].reshape(E * H, I)).reshape(E, H, I // 2)),
        dev(_tile(dn[1].reshape(E * H, I // 16), I)), dev(dn[2]), None, ws)
    assert metis.metis_check_device_status() == 0
    off = lambda name: metis.metis_moe_nvfp4_workspace_offset(name, T, k, E, H, I)
    Sp = (T * k + 127 * E + 127) // 128 * 128
    o_dev = _region(ws, off("O"), Sp * H, torch.bfloat16)
    s2r_dev = _region(ws, off("SLOT_TO_ROW"), T * k, torch.int32)
    assert_bytes_equal(s2r_dev.cpu().numpy(), g["s2r"], "routing of the y=NULL run")
    wu, wd = _shared_weights(25, H, I_s)
    y, hs = _run_fused(metis, d, wu, wd, o_dev, s2r_dev)
    _check_fused(d, wu, wd, y, hs, _o_slots(g, g["s2r"], T, k))
    z = np.zeros_like(wu), np.zeros_like(wd)
    y0, _ = _run_fused(metis, d, z[0], z[1], o_dev, s2r_dev)
    assert_bytes_equal(y0, g["y"], "zero shared expert = routed combine")


def _tile(sf, K):
    from test_gpu_nvfp4 import tile_np
    return tile_np(sf, K)


def test_shared_fused_combine_full_size(metis):
    """4096 tokens, hidden 2048, latent 1024 (routed and shared), 64 experts,
    top-8: the FP8 routed layer with y = NULL, then the fused shared combine;
    sampled tokens."""
    d = synth.moe()
    T, H, I, E, k = d["T"], d["H"], d["I"], d["E"], d["topk"]
    g = run_moe(metis, d)
    o_dev = dev(g["o"].view(np.int16)).view(torch.bfloat16)
    wu, wd = _shared_weights(26, H, 1024)
    y, hs = _run_fused(metis, d, wu, wd, o_dev, dev(g["s2r"]))
    rng = np.random.default_rng(3)
    toks = np.unique(np.r_[rng.choice(T, 24, replace=False), 0, T - 1])
    _check_fused(d, wu, wd, y, hs, _o_slots(g, g["s2r"], T, k), tokens=toks)
