"""GPU parity of the quantizers, the W8A8 GEMM and the W8A16 GEMM against the
CPU oracle, through the C ABI. Bytes and scales bit-exact; BF16 outputs within
1e-2 * (1 + |ref|)."""
import numpy as np
import pytest
import torch

import oracle
from moe_gemm_token_b200 import synth
from gpu_helpers import assert_bytes_equal, assert_close, bf16_dev, bf16_host, dev

pytestmark = pytest.mark.gpu


def _quant_gpu(m, x_bits, ldx=None):
    M, K = x_bits.shape
    if ldx is None:
        xd = bf16_dev(x_bits)
    else:
        big = np.zeros((M, ldx), dtype=np.uint16)
        big[:, :K] = x_bits
        xd = bf16_dev(big)[:, :K]
    xq = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    s = torch.empty((M,), dtype=torch.float32, device="cuda")
    m.metis_quant_fp8_per_token(xd, xq, s)
    torch.cuda.synchronize()
    return xq.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("M,K,seed", [(16, 256, 0), (37, 264, 1), (5, 6144, 2), (3, 20480, 3),
                                      (1, 8, 4), (200, 2048, 5), (9, 16384, 6), (130, 1024, 7)])
def test_quant_per_token_bit_exact(metis, M, K, seed):
    d = synth.linear(seed, M, K, 8, outlier_channels=min(4, K), outlier_scale=25.0,
                     zero_rows=(M // 2,), row_magnitude_log10=(-3, 3))
    q, s = _quant_gpu(metis, d["x"])
    qr, sr = oracle.quant_per_token(d["x"])
    assert_bytes_equal(s.view(np.uint32), sr.view(np.uint32), "scales")
    assert_bytes_equal(q, qr, "codes")


def test_quant_per_token_extremes(metis):
    """BF16 subnormal rows (448/amax overflows and is clamped), huge rows,
    negative zeros, exact ties of the E4M3 grid."""
    K = 64
    rows = [
        np.full(K, 2.0 ** -130, np.float32),                       # subnormal BF16
        np.linspace(-3e38, 3e38, K).astype(np.float32),           # near BF16 max
        np.where(np.arange(K) % 2 == 0, -0.0, 0.0).astype(np.float32),
        (np.arange(K) - 32).astype(np.float32) * 0.5,              # many exact ties after scaling
        np.r_[448.0, np.full(K - 1, 1.0625, np.float32)].astype(np.float32),
        np.r_[np.full(K - 1, 1e-8, np.float32), 1.0].astype(np.float32),
    ]
    x = synth.f32_to_bf16_bits(np.stack(rows))
    q, s = _quant_gpu(metis, x)
    qr, sr = oracle.quant_per_token(x)
    assert_bytes_equal(s.view(np.uint32), sr.view(np.uint32), "scales")
    assert_bytes_equal(q, qr, "codes")


def test_quant_per_token_strided(metis):
    d = synth.linear(3, 50, 1000, 8, outlier_channels=3, outlier_scale=30.0)
    q, s = _quant_gpu(metis, d["x"], ldx=1032)
    qr, sr = oracle.quant_per_token(d["x"])
    assert_bytes_equal(q, qr, "codes")
    assert_bytes_equal(s.view(np.uint32), sr.view(np.uint32), "scales")


@pytest.mark.parametrize("N,K", [(512, 256), (33, 100), (7, 20484), (1000, 4096)])
def test_quant_per_channel_bit_exact(metis, N, K):
    rng = np.random.default_rng(N + K)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[N // 3] = 0.0
    wd = dev(w)
    wq = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    s = torch.empty((N,), dtype=torch.float32, device="cuda")
    metis.metis_quant_fp8_per_channel(wd, wq, s)
    torch.cuda.synchronize()
    qr, sr = oracle.quant_per_channel(w)
    assert_bytes_equal(s.cpu().numpy().view(np.uint32), sr.view(np.uint32), "scales")
    assert_bytes_equal(wq.cpu().numpy(), qr, "codes")


def _prep_weights(metis, w):
    N, K = w.shape
    wq = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    s = torch.empty((N,), dtype=torch.float32, device="cuda")
    metis.metis_quant_fp8_per_channel(dev(w), wq, s)
    return wq, s


@pytest.mark.parametrize("M,N,K", [(16, 512, 256), (300, 520, 272), (1, 8, 16), (129, 264, 1040),
                                   (520, 784, 1024), (257, 1024, 2048), (4500, 520, 256),
                                   # the final partial wave cut into column quarters on 74
                                   # CTA pairs: 384 tiles (14 in the last wave); 76 tiles with
                                   # ragged M and N (2); 84 tiles whose last tile column is
                                   # 64 wide, so two of its quarters fall past N (10)
                                   (4096, 6144, 256), (1000, 4808, 256), (1536, 3392, 384)])
def test_fp8_gemm_parity(metis, M, N, K):
    d = synth.linear(M * 7 + N, M, K, N, outlier_channels=4, outlier_scale=20.0, zero_rows=(M // 3,))
    wq, s_w = _prep_weights(metis, d["w"])
    xd = bf16_dev(d["x"])
    xq = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    s_tok = torch.empty((M,), dtype=torch.float32, device="cuda")
    metis.metis_quant_fp8_per_token(xd, xq, s_tok)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_fp8_gemm(xq, metis.METIS_A_E4M3, s_tok, wq, s_w, y)
    assert metis.metis_check_device_status() == 0
    wq_r, sw_r = oracle.quant_per_channel(d["w"])
    assert_bytes_equal(wq.cpu().numpy(), wq_r, "weight codes")
    y_r, y64, xq_r, st_r = oracle.linear_w8a8(d["x"], wq_r, sw_r)
    assert_bytes_equal(xq.cpu().numpy(), xq_r, "activation codes")
    assert_close(bf16_host(y), y64, f"y {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(200, 272, 512), (4096, 6144, 64)])
def test_fp8_gemm_exact_integer_products(metis, M, N, K):
    """Codes whose products and sums are small integers: the FP32 accumulation
    is exact, so with unit scales the output equals the oracle's BF16 bits
    (4096 x 6144: every column piece of the final wave lands where it belongs)."""
    rng = np.random.default_rng(11)
    vals = np.array([0x38, 0x40, 0x44, 0xB8, 0xC0, 0x00, 0x30], np.uint8)  # 1,2,3,-1,-2,0,0.5
    a = vals[rng.integers(0, vals.size, (M, K))]
    b = vals[rng.integers(0, vals.size, (N, K))]
    one_m, one_n = np.ones(M, np.float32), np.ones(N, np.float32)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_fp8_gemm(dev(a), 0, dev(one_m), dev(b), dev(one_n), y)
    yr, _ = oracle.gemm_w8a8(a, one_m, b, one_n)
    assert_bytes_equal(bf16_host(y), yr, "bf16 bits")


def _fused(metis, xd, wq, s_w, M, N, K):
    ws = torch.empty((metis.metis_workspace_size(metis.METIS_OP_FP8_GEMM_FUSED, M, N, K, 0, 0),),
                     dtype=torch.uint8, device="cuda")
    s_tok = torch.full((M,), float("nan"), dtype=torch.float32, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_fp8_gemm(xd, metis.METIS_A_BF16, s_tok, wq, s_w, y, workspace=ws)
    assert metis.metis_check_device_status() == 0
    return y, s_tok


@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (16, 512, 256), (100, 264, 208), (128, 256, 128),
                                   (129, 264, 1040), (300, 520, 272), (520, 784, 1024),
                                   (257, 1024, 2048), (300, 264, 20480)])
def test_fp8_gemm_fused_parity(metis, M, N, K):
    """BF16 A quantized inside the GEMM (a_kind = BF16): the scales equal the
    standalone quantizer's and the oracle's bit for bit; y is within tolerance
    of the oracle and identical to the unfused GEMM on the standalone codes
    (same codes in shared memory, same accumulation order)."""
    d = synth.linear(M * 5 + N + K, M, K, N, outlier_channels=4, outlier_scale=20.0,
                     zero_rows=(M // 3,))
    wq, s_w = _prep_weights(metis, d["w"])
    xd = bf16_dev(d["x"])
    xq = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    s1 = torch.empty((M,), dtype=torch.float32, device="cuda")
    metis.metis_quant_fp8_per_token(xd, xq, s1)
    y1 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_fp8_gemm(xq, metis.METIS_A_E4M3, s1, wq, s_w, y1)
    y2, s2 = _fused(metis, xd, wq, s_w, M, N, K)
    wq_r, sw_r = oracle.quant_per_channel(d["w"])
    _, y64, _, st_r = oracle.linear_w8a8(d["x"], wq_r, sw_r)
    assert_bytes_equal(s2.cpu().numpy().view(np.uint32), st_r.view(np.uint32), "fused s_tok")
    assert_close(bf16_host(y2), y64, f"fused y {M}x{N}x{K}")
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), "fused != unfused"


def test_fp8_gemm_fused_extremes(metis):
    """Rows near the ends of the BF16 range, all-zero rows and rows with one
    non-zero element go through the in-kernel quantization like the
    standalone quantizer (saturation, zero scale)."""
    rng = np.random.default_rng(23)
    M, N, K = 160, 264, 384
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[0] *= 1.0e35 / np.abs(x[0]).max()        # huge scale, y still representable in BF16
    x[1] *= 1.0e-38                            # tiny, partly subnormal after scaling
    x[2] = 0.0
    x[3] = 0.0
    x[3, 17] = -2.5
    x[150:] *= 1000.0                          # the second 128-row block
    xb = synth.f32_to_bf16_bits(x)
    w = rng.standard_normal((N, K)).astype(np.float32)
    wq, s_w = _prep_weights(metis, w)
    y2, s2 = _fused(metis, bf16_dev(xb), wq, s_w, M, N, K)
    wq_r, sw_r = oracle.quant_per_channel(w)
    _, y64, _, st_r = oracle.linear_w8a8(xb, wq_r, sw_r)
    assert_bytes_equal(s2.cpu().numpy().view(np.uint32), st_r.view(np.uint32), "fused s_tok")
    assert np.all(bf16_host(y2)[2] == 0)
    assert_close(bf16_host(y2), y64, "fused extremes")


def test_linear_fast_math(metis):
    """M > 8 with fast_math: the per-token quantizer, then the E4M3 GEMM; the
    result equals the two direct calls and the fused variant bit for bit."""
    M, N, K = 64, 256, 512
    d = synth.linear(22, M, K, N)
    wq, s_w = _prep_weights(metis, d["w"])
    xd = bf16_dev(d["x"])
    y1, s1 = _fused(metis, xd, wq, s_w, M, N, K)
    ws = torch.empty((metis.metis_workspace_size(metis.METIS_OP_LINEAR, M, N, K, 0, 0),),
                     dtype=torch.uint8, device="cuda")
    s2 = torch.empty((M,), dtype=torch.float32, device="cuda")
    y2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_linear(xd, wq, s_w, y2, fast_math=True, s_tok=s2, workspace=ws)
    xq = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    s3 = torch.empty((M,), dtype=torch.float32, device="cuda")
    y3 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_quant_fp8_per_token(xd, xq, s3)
    metis.metis_fp8_gemm(xq, metis.METIS_A_E4M3, s3, wq, s_w, y3)
    torch.cuda.synchronize()
    assert torch.equal(y2.view(torch.int16), y3.view(torch.int16))
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(s1, s2) and torch.equal(s2, s3)
    assert torch.equal(ws[:M * K].view(M, K), xq)
    # without fast-math the default maths (W8A16) runs, bit-identical to the direct call
    y4 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    y5 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_linear(xd, wq, s_w, y4, fast_math=False, s_tok=s2, workspace=ws)
    metis.metis_w8a16_gemm(xd, wq, s_w, y5)
    torch.cuda.synchronize()
    assert torch.equal(y4.view(torch.int16), y5.view(torch.int16))


@pytest.mark.parametrize("M,N,K", [(1, 1000, 4096), (2, 37, 272), (3, 300, 12288), (4, 1000, 4096),
                                   (5, 48, 1024), (8, 1000, 4096), (8, 16, 16), (7, 2333, 1040),
                                   (6, 148 * 16 * 7 + 5, 2048), (8, 3000, 8192), (1, 64, 12288),
                                   (8, 57344, 4096), (3, 777, 2560), (8, 100, 3072), (1, 5, 1024),
                                   (8, 9, 2048), (2, 148 * 8 + 3, 4096)])
def test_w8a16_parity(metis, M, N, K):
    d = synth.linear(M + 13 * N + K, M, K, N)
    wq, s_w = _prep_weights(metis, d["w"])
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_w8a16_gemm(bf16_dev(d["x"]), wq, s_w, y)
    torch.cuda.synchronize()
    wq_r, sw_r = oracle.quant_per_channel(d["w"])
    assert_bytes_equal(wq.cpu().numpy(), wq_r, "weight codes")
    _, y64 = oracle.gemm_w8a16(d["x"], wq_r, sw_r)
    assert_close(bf16_host(y), y64, f"w8a16 {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(9, 264, 512), (64, 256, 128), (100, 520, 272), (128, 128, 64),
                                   (200, 1000, 1040), (300, 6144, 2048), (513, 136, 4096),
                                   # enough tiles for 256-token tiles (one wave instead of two)
                                   (1000, 4104, 1040), (1500, 2056, 256)])
def test_w8a16_tensor_core_parity(metis, M, N, K):
    """M > 8: the default maths on the tensor cores (weights widened to BF16
    in tensor memory, x BF16 from shared memory), ragged in M, N and K, on
    128-token tiles and (the last two shapes) 256-token tiles."""
    d = synth.linear(M * 3 + N + 7 * K, M, K, N, outlier_channels=2, outlier_scale=20.0)
    wq, s_w = _prep_weights(metis, d["w"])
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_w8a16_gemm(bf16_dev(d["x"]), wq, s_w, y)
    assert metis.metis_check_device_status() == 0
    wq_r, sw_r = oracle.quant_per_channel(d["w"])
    _, y64 = oracle.gemm_w8a16(d["x"], wq_r, sw_r)
    assert_close(bf16_host(y), y64, f"w8a16 tensor {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(160, 264, 320), (1200, 2056, 384)])
def test_w8a16_tensor_core_exact_products(metis, M, N, K):
    """Every weight code an E4M3 subnormal or small normal and x small
    integers: products and partial sums are exact in FP32, so the output
    equals the oracle's BF16 bits. A widening that lost subnormals, or a
    wrong lane/column layout of the weights in tensor memory, fails here
    (the second shape on 256-token tiles)."""
    rng = np.random.default_rng(9)
    codes = (rng.integers(1, 8, (N, K)) | (rng.integers(0, 2, (N, K)) << 7)).astype(np.uint8)
    codes[:, ::5] = 0x38  # 1.0
    codes[::3, 1::7] = 0xC0  # -2.0
    x = synth.f32_to_bf16_bits(rng.integers(-4, 5, (M, K)).astype(np.float32))
    s_w = np.ones(N, np.float32)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_w8a16_gemm(bf16_dev(x), dev(codes), dev(s_w), y)
    assert metis.metis_check_device_status() == 0
    yr, _ = oracle.gemm_w8a16(x, codes, s_w)
    assert np.any(yr != 0)
    assert_bytes_equal(bf16_host(y), yr, "w8a16 tensor exact")


def test_w8a16_tensor_core_nan_codes(metis):
    """E4M3 NaN weight codes (0x7F, 0xFF) widen to NaN: every output of those
    channels is NaN, and every other output matches the oracle."""
    M, N, K = 272, 520, 192
    d = synth.linear(77, M, K, N, outlier_channels=0, outlier_scale=1.0)
    wq_r, sw_r = oracle.quant_per_channel(d["w"])
    wq_r = wq_r.copy()
    wq_r[3, 5] = 0x7F
    wq_r[300, 191] = 0xFF
    wq_r[519, 0] = 0x7F
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_w8a16_gemm(bf16_dev(d["x"]), dev(wq_r), dev(sw_r), y)
    assert metis.metis_check_device_status() == 0
    got = bf16_host(y)
    nan = (got & 0x7FFF) > 0x7F80
    assert np.array_equal(np.nonzero(nan.any(axis=0))[0], [3, 300, 519])
    assert nan[:, [3, 300, 519]].all()
    keep = np.setdiff1d(np.arange(N), [3, 300, 519])
    _, y64 = oracle.gemm_w8a16(d["x"], wq_r[keep], sw_r[keep])
    assert_close(got[:, keep], y64, "w8a16 tensor, finite channels")


def _widened_ws(metis, M, N, K):
    n = metis.metis_workspace_size(metis.METIS_OP_W8A16_WIDENED, M, N, K)
    return torch.zeros((n,), dtype=torch.uint8, device="cuda")


def test_w8a16_widening_is_exact_for_every_code(metis):
    """The widening pass writes the BF16 value of every E4M3 code exactly
    (subnormals included) and a same-signed NaN for 0x7F and 0xFF."""
    N, K = 16, 256
    # every code in every row, at a different column per row
    codes = ((np.arange(K)[None, :] + 17 * np.arange(N)[:, None]) % 256).astype(np.uint8)
    ws = _widened_ws(metis, 9, N, K)
    x = torch.zeros((9, K), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((9, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_w8a16_gemm_widened(x, dev(codes), dev(np.ones(N, np.float32)), y, ws)
    assert metis.metis_check_device_status() == 0
    wb = ws[:2 * N * K].view(torch.int16).view(N, K).cpu().numpy().view(np.uint16)
    want = oracle.e4m3_decode(codes)
    isnan = np.isnan(want)
    assert np.array_equal(isnan, (codes & 0x7F) == 0x7F)
    got = oracle.bf16_to_float(wb).astype(np.float64)
    assert np.array_equal(got[~isnan], want[~isnan])
    assert np.array_equal(np.signbit(got[~isnan]), np.signbit(want[~isnan]))  # -0 stays -0
    assert np.all(np.isnan(got[isnan]))
    assert np.array_equal(np.signbit(got[isnan]), (codes[isnan] & 0x80) != 0)


@pytest.mark.parametrize("M,N,K", [(9, 264, 512), (256, 256, 128), (300, 6144, 2048), (513, 136, 4096),
                                   (1000, 520, 1040), (129, 8, 16), (4500, 264, 256)])
def test_w8a16_widened_parity(metis, M, N, K):
    """The default maths through widened weights and the BF16 CTA-pair GEMM
    (per-channel scale in its epilogue), ragged in M, N and K."""
    d = synth.linear(M * 5 + N + 3 * K, M, K, N, outlier_channels=2, outlier_scale=20.0)
    wq, s_w = _prep_weights(metis, d["w"])
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_w8a16_gemm_widened(bf16_dev(d["x"]), wq, s_w, y, _widened_ws(metis, M, N, K))
    assert metis.metis_check_device_status() == 0
    wq_r, sw_r = oracle.quant_per_channel(d["w"])
    _, y64 = oracle.gemm_w8a16(d["x"], wq_r, sw_r)
    assert_close(bf16_host(y), y64, f"w8a16 widened {M}x{N}x{K}")


def test_w8a16_widened_exact_products(metis):
    """Subnormal and small normal weight codes, small-integer x, unit scales:
    every product and partial sum is exact in FP32, so the BF16 outputs equal
    the oracle's bit for bit."""
    rng = np.random.default_rng(19)
    M, N, K = 300, 264, 320
    codes = (rng.integers(1, 8, (N, K)) | (rng.integers(0, 2, (N, K)) << 7)).astype(np.uint8)
    codes[:, ::5] = 0x38  # 1.0
    codes[::3, 1::7] = 0xC0  # -2.0
    x = synth.f32_to_bf16_bits(rng.integers(-4, 5, (M, K)).astype(np.float32))
    s_w = np.ones(N, np.float32)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_w8a16_gemm_widened(bf16_dev(x), dev(codes), dev(s_w), y, _widened_ws(metis, M, N, K))
    assert metis.metis_check_device_status() == 0
    yr, _ = oracle.gemm_w8a16(x, codes, s_w)
    assert np.any(yr != 0)
    assert_bytes_equal(bf16_host(y), yr, "w8a16 widened exact")


def test_w8a16_widened_nan_codes(metis):
    M, N, K = 272, 520, 192
    d = synth.linear(78, M, K, N)
    wq_r, sw_r = oracle.quant_per_channel(d["w"])
    wq_r = wq_r.copy()
    wq_r[3, 5] = 0x7F
    wq_r[300, 191] = 0xFF
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_w8a16_gemm_widened(bf16_dev(d["x"]), dev(wq_r), dev(sw_r), y, _widened_ws(metis, M, N, K))
    assert metis.metis_check_device_status() == 0
    got = bf16_host(y)
    nan = (got & 0x7FFF) > 0x7F80
    assert np.array_equal(np.nonzero(nan.any(axis=0))[0], [3, 300])
    assert nan[:, [3, 300]].all()
    keep = np.setdiff1d(np.arange(N), [3, 300])
    _, y64 = oracle.gemm_w8a16(d["x"], wq_r[keep], sw_r[keep])
    assert_close(got[:, keep], y64, "w8a16 widened, finite channels")


WIDEN_MIN_TOKENS = 2048  # metis_linear widens the weights into the workspace from here


@pytest.mark.parametrize("M", [300, 2047, 2048, 2100])
def test_linear_default_maths_dispatch(metis, M):
    """metis_linear without fast-math: M >= 2048 with a large enough
    workspace runs the widened-weights GEMM, otherwise the in-kernel
    widening; each is bit-identical to its direct call."""
    N, K = 384, 512
    d = synth.linear(M + 11, M, K, N)
    wq, s_w = _prep_weights(metis, d["w"])
    x = bf16_dev(d["x"])
    ws = _widened_ws(metis, M, N, K)
    y_lin = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    y_dir = torch.empty_like(y_lin)
    metis.metis_linear(x, wq, s_w, y_lin, fast_math=False, workspace=ws)
    if M >= WIDEN_MIN_TOKENS:
        metis.metis_w8a16_gemm_widened(x, wq, s_w, y_dir, _widened_ws(metis, M, N, K))
    else:
        metis.metis_w8a16_gemm(x, wq, s_w, y_dir)
    assert metis.metis_check_device_status() == 0
    assert torch.equal(y_lin.view(torch.int16), y_dir.view(torch.int16))
    # without a workspace the in-kernel path runs at any M
    y_in = torch.empty_like(y_lin)
    metis.metis_linear(x, wq, s_w, y_in, fast_math=False)
    y_ref = torch.empty_like(y_lin)
    metis.metis_w8a16_gemm(x, wq, s_w, y_ref)
    torch.cuda.synchronize()
    assert torch.equal(y_in.view(torch.int16), y_ref.view(torch.int16))


def test_w8a16_subnormal_weights_and_wide_x(metis):
    """Weight rows with many E4M3 subnormal codes and tokens whose elements
    span many binades: the widening and the per-token shift stay exact."""
    rng = np.random.default_rng(5)
    M, N, K = 8, 96, 512
    w = (rng.standard_normal((N, K)) * np.power(10.0, rng.uniform(-5, 0, (N, K)))).astype(np.float32)
    x = (rng.standard_normal((M, K)) * np.power(10.0, rng.uniform(-4, 4, (M, K)))).astype(np.float32)
    x[3] = 0.0
    xb = synth.f32_to_bf16_bits(x)
    wq, s_w = _prep_weights(metis, w)
    wq_r, sw_r = oracle.quant_per_channel(w)
    assert np.mean((wq_r & 0x78) == 0) > 0.2  # plenty of subnormal / zero codes
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_w8a16_gemm(bf16_dev(xb), wq, s_w, y)
    torch.cuda.synchronize()
    _, y64 = oracle.gemm_w8a16(xb, wq_r, sw_r)
    assert_close(bf16_host(y), y64, "w8a16 subnormal weights")


def test_linear_dispatch(metis):
    """M <= 8 takes the default maths (W8A16), bit-identical to the direct call."""
    d = synth.linear(21, 4, 512, 64)
    wq, s_w = _prep_weights(metis, d["w"])
    y1 = torch.empty((4, 64), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty_like(y1)
    metis.metis_w8a16_gemm(bf16_dev(d["x"]), wq, s_w, y1)
    metis.metis_linear(bf16_dev(d["x"]), wq, s_w, y2, fast_math=True)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_w8a16_all_subnormal_codes_exact(metis):
    """Every weight code is an E4M3 subnormal (+-m * 2^-9) and x holds small
    integers, so every product and partial sum is exact in FP32: the output
    must equal the oracle's BF16 bits. A widening that lost E4M3 subnormals
    would return zeros here."""
    rng = np.random.default_rng(8)
    M, N, K = 8, 64, 256
    codes = (rng.integers(1, 8, (N, K)) | (rng.integers(0, 2, (N, K)) << 7)).astype(np.uint8)
    x = synth.f32_to_bf16_bits(rng.integers(-4, 5, (M, K)).astype(np.float32))
    s_w = np.ones(N, np.float32)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    metis.metis_w8a16_gemm(bf16_dev(x), dev(codes), dev(s_w), y)
    torch.cuda.synchronize()
    yr, _ = oracle.gemm_w8a16(x, codes, s_w)
    assert np.any(yr != 0)
    assert_bytes_equal(bf16_host(y), yr, "w8a16 subnormal codes")
