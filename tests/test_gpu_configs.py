"""GPU parity at the full sizes of the five workloads, in the launch
configuration the benchmark times. Bytes are compared in full. BF16 outputs
are compared in full for the tiny layer, the 4096-token prefill chain (both
maths), decode and the 4096-token routed-expert layer; for the large-M sweep
(up to 2.2 TFLOP per GEMM) on 256 sampled rows that the oracle computes one by
one, always including the extreme rows (largest and smallest magnitudes)."""
import numpy as np
import pytest
import torch

import oracle
from moe_gemm_token_b200 import synth
from gpu_helpers import assert_bytes_equal, assert_close, bf16_dev, bf16_host, dev
from test_gpu_moe import check_moe, run_moe

pytestmark = pytest.mark.gpu


def _weights(metis, w):
    N, K = w.shape
    wq = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    s = torch.empty((N,), dtype=torch.float32, device="cuda")
    metis.metis_quant_fp8_per_channel(dev(w), wq, s)
    torch.cuda.synchronize()
    wq_r, s_r = oracle.quant_per_channel(w)
    assert_bytes_equal(wq.cpu().numpy(), wq_r, "weight codes")
    assert_bytes_equal(s.cpu().numpy().view(np.uint32), s_r.view(np.uint32), "weight scales")
    return wq, s, wq_r, s_r


def _sample_rows(M, x_bits, n=48, seed=0):
    x = synth.bf16_bits_to_f32(x_bits)
    amax = np.abs(x).max(axis=1)
    rng = np.random.default_rng(seed)
    extra = [int(np.argmax(amax)), int(np.argmin(amax)), 0, M - 1]
    return np.unique(np.r_[rng.choice(M, n, replace=False), extra]).astype(np.int64)


def test_tiny_linear_full(metis):
    d = synth.tiny_linear()
    wq, s_w, wq_r, s_r = _weights(metis, d["w"])
    xq = torch.empty((16, 256), dtype=torch.uint8, device="cuda")
    s_tok = torch.empty((16,), dtype=torch.float32, device="cuda")
    metis.metis_quant_fp8_per_token(bf16_dev(d["x"]), xq, s_tok)
    y = torch.empty((16, 512), dtype=torch.bfloat16, device="cuda")
    metis.metis_fp8_gemm(xq, 0, s_tok, wq, s_w, y)
    torch.cuda.synchronize()
    y_r, y64, xq_r, st_r = oracle.linear_w8a8(d["x"], wq_r, s_r)
    assert_bytes_equal(xq.cpu().numpy(), xq_r, "codes")
    assert s_tok.cpu().numpy()[7] == 0.0
    assert_close(bf16_host(y), y64, "tiny")
    assert np.all(bf16_host(y)[7] & 0x7FFF == 0)  # the all-zero token gives zeros


def test_prefill_chain_full_size(metis):
    d = synth.prefill_chain()
    M, K, N = d["M"], d["K"], d["N"]
    w1, s1, w1r, s1r = _weights(metis, d["w1"])
    w2, s2, w2r, s2r = _weights(metis, d["w2"])
    xq1 = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    st1 = torch.empty((M,), dtype=torch.float32, device="cuda")
    y1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    xq2 = torch.empty((M, N), dtype=torch.uint8, device="cuda")
    st2 = torch.empty((M,), dtype=torch.float32, device="cuda")
    y2 = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    metis.metis_quant_fp8_per_token(bf16_dev(d["x"]), xq1, st1)
    metis.metis_fp8_gemm(xq1, 0, st1, w1, s1, y1)
    metis.metis_quant_fp8_per_token(y1, xq2, st2)
    metis.metis_fp8_gemm(xq2, 0, st2, w2, s2, y2)
    assert metis.metis_check_device_status() == 0
    xq1r, st1r = oracle.quant_per_token(d["x"])
    assert_bytes_equal(xq1.cpu().numpy(), xq1r, "layer-1 codes")
    assert_bytes_equal(st1.cpu().numpy().view(np.uint32), st1r.view(np.uint32), "layer-1 scales")
    # every token of both layers
    _, y1_64 = oracle.gemm_w8a8(xq1r, st1r, w1r, s1r)
    y1h = bf16_host(y1)
    assert_close(y1h, y1_64, "layer 1")
    del y1_64
    # layer 2 starts from the GPU's own layer-1 output
    xq2r, st2r = oracle.quant_per_token(y1h)
    assert_bytes_equal(xq2.cpu().numpy(), xq2r, "layer-2 codes")
    assert_bytes_equal(st2.cpu().numpy().view(np.uint32), st2r.view(np.uint32), "layer-2 scales")
    _, y2_64 = oracle.gemm_w8a8(xq2r, st2r, w2r, s2r)
    assert_close(bf16_host(y2), y2_64, "layer 2")


@pytest.mark.parametrize("widened", [False, True])
def test_prefill_chain_default_maths_full_size(metis, widened):
    """The same 4096-token chain through the default maths (metis_linear
    without fast-math: W8A16, weights widened to BF16 in the kernel, or first
    into a workspace for the BF16 CTA-pair GEMM)."""
    d = synth.prefill_chain()
    M, K, N = d["M"], d["K"], d["N"]
    w1, s1, w1r, s1r = _weights(metis, d["w1"])
    w2, s2, w2r, s2r = _weights(metis, d["w2"])
    y1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    s_tok = torch.empty((M,), dtype=torch.float32, device="cuda")
    ws = None
    if widened:
        n = metis.metis_workspace_size(metis.METIS_OP_W8A16_WIDENED, M, N, K)
        ws = torch.empty((n,), dtype=torch.uint8, device="cuda")
    metis.metis_linear(bf16_dev(d["x"]), w1, s1, y1, fast_math=False, s_tok=s_tok, workspace=ws)
    metis.metis_linear(y1, w2, s2, y2, fast_math=False, s_tok=s_tok, workspace=ws)
    assert metis.metis_check_device_status() == 0
    # every token of both layers
    _, y1_64 = oracle.gemm_w8a16(d["x"], w1r, s1r)
    y1h = bf16_host(y1)
    assert_close(y1h, y1_64, "layer 1 (default maths)")
    del y1_64
    _, y2_64 = oracle.gemm_w8a16(y1h, w2r, s2r)
    assert_close(bf16_host(y2), y2_64, "layer 2 (default maths)")


@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_decode_full_size(metis, M):
    d = synth.decode(M=M)
    wq, s_w, wq_r, s_r = _weights(metis, d["w"])
    y = torch.empty((M, d["N"]), dtype=torch.bfloat16, device="cuda")
    metis.metis_w8a16_gemm(bf16_dev(d["x"]), wq, s_w, y)
    assert metis.metis_check_device_status() == 0
    _, y64 = oracle.gemm_w8a16(d["x"], wq_r, s_r)
    assert_close(bf16_host(y), y64, f"decode M={M}")


def test_moe_full_size(metis):
    """All 4096 tokens (32768 routed slots), every stage."""
    d = synth.moe()
    g = run_moe(metis, d)
    check_moe(d, g)


@pytest.mark.parametrize("M,K", [(8192, 4096), (16384, 4096), (8192, 8192), (16384, 8192)])
def test_large_m_full_size(metis, M, K):
    d = synth.large_m(M=M, K=K)
    N = K
    wq, s_w, wq_r, s_r = _weights(metis, d["w"])
    xq = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    st = torch.empty((M,), dtype=torch.float32, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    x_dev = bf16_dev(d["x"])
    metis.metis_quant_fp8_per_token(x_dev, xq, st)
    metis.metis_fp8_gemm(xq, 0, st, wq, s_w, y)
    assert metis.metis_check_device_status() == 0
    xq_r, st_r = oracle.quant_per_token(d["x"])
    assert_bytes_equal(xq.cpu().numpy(), xq_r, "codes")
    assert_bytes_equal(st.cpu().numpy().view(np.uint32), st_r.view(np.uint32), "scales")
    rows = _sample_rows(M, d["x"], n=256)  # 256 sampled rows and the extreme ones
    _, y64 = oracle.gemm_w8a8(xq_r, st_r, wq_r, s_r, rows=rows)
    assert_close(bf16_host(y)[rows], y64, f"large M {M}x{K}")
    # the fused-quantization prologue on the same input: the same scales and,
    # bit for bit, the same output as quantizer + E4M3 GEMM
    st_f = torch.empty_like(st)
    y_f = torch.empty_like(y)
    ws = torch.empty((metis.metis_workspace_size(metis.METIS_OP_FP8_GEMM_FUSED, M, N, K),),
                     dtype=torch.uint8, device="cuda")
    metis.metis_fp8_gemm(x_dev, metis.METIS_A_BF16, st_f, wq, s_w, y_f, workspace=ws)
    assert metis.metis_check_device_status() == 0
    assert_bytes_equal(st_f.cpu().numpy().view(np.uint32), st_r.view(np.uint32), "fused scales")
    assert torch.equal(y_f.view(torch.int16), y.view(torch.int16)), "fused prologue differs"
