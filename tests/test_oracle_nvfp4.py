"""Pins of the oracle's NVFP4 functions ("Lernex/Metis-1.6-Praxis-NVFP4", "What
is in NVFP4": E2M1 values, one E4M3 scale per 16 inputs, one FP32 scale per
expert; "What --fast-math does": the experts' inputs rounded to FP4 too).

Each check comes from outside the oracle's own code: the E2M1 format's bit
fields, the round-to-nearest-even rule on a brute-force grid, exact round
trips of data built from representable parts, the error bound of the format,
and a float64 numpy matmul of the decoded operands.
"""
import numpy as np
import pytest

import oracle


def _e2m1_from_bits(c):
    # sign | 2 exponent bits (bias 1) | 1 mantissa bit; exponent 0 is subnormal
    s = -1.0 if c & 8 else 1.0
    e = (c >> 1) & 3
    m = c & 1
    return s * (0.5 * m if e == 0 else 2.0 ** (e - 1) * (1.0 + 0.5 * m))


def test_e2m1_decode_matches_bit_fields():
    got = oracle.e2m1_decode(np.arange(16, dtype=np.uint8))
    want = np.array([_e2m1_from_bits(c) for c in range(16)])
    assert np.array_equal(got, want)
    # the magnitudes the OCP microscaling format lists for FP4 (E2M1)
    assert list(got[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_encode_round_trip_and_ties():
    vals = oracle.e2m1_decode(np.arange(16, dtype=np.uint8)).astype(np.float32)
    codes = oracle.e2m1_encode(vals)
    assert np.array_equal(oracle.e2m1_decode(codes), vals.astype(np.float64))
    # midpoints go to the code with an even last bit
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    assert list(oracle.e2m1_decode(oracle.e2m1_encode(mids))) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    assert list(oracle.e2m1_decode(oracle.e2m1_encode(-mids))) == [-0.0, -1.0, -1.0, -2.0, -2.0,
                                                                    -4.0, -4.0]
    # saturation, no NaN or infinity in the format
    big = np.array([6.0, 6.5, 7.0, 1e30, np.inf], dtype=np.float32)
    assert np.all(oracle.e2m1_encode(big) == 7)
    assert np.all(oracle.e2m1_encode(-big) == 15)


def test_e2m1_encode_is_nearest_on_a_grid():
    v = np.linspace(-7.0, 7.0, 20001).astype(np.float32)
    got = oracle.e2m1_decode(oracle.e2m1_encode(v))
    grid = np.array([_e2m1_from_bits(c) for c in range(16)])
    dist = np.abs(v.astype(np.float64)[:, None] - grid[None, :])
    best = dist.min(axis=1)
    assert np.all(np.abs(got - v) == best)
    # monotone
    assert np.all(np.diff(got) >= 0)


def test_nvfp4_quant_exact_round_trip():
    # data built from representable parts: g = 2^-3 so that amax/2688 = g,
    # every block holds a +-6 code, so block amax / (6 g) = its scale exactly
    rng = np.random.default_rng(11)
    R, K = 6, 96
    q = rng.integers(0, 16, size=(R, K)).astype(np.uint8)
    q[:, ::16] = rng.choice([7, 15], size=(R, K // 16))
    sb = rng.integers(0x08, 0x7E, size=(R, K // 16)).astype(np.uint8)
    sb[:, 0] = 0x7E  # 448: the row maximum lives in block 0
    g = np.float32(0.125)
    x = oracle.nvfp4_dequant(q, sb, np.full(R, g)).astype(np.float32)
    q2, sb2, g2 = oracle.nvfp4_quant(x, per_row=True)
    assert np.all(g2 == g)
    assert np.array_equal(sb2, sb)
    # +-0 may differ in sign only where the value is zero
    assert np.array_equal(oracle.e2m1_decode(q2), oracle.e2m1_decode(q))
    # the same matrix with one global scale
    q3, sb3, g3 = oracle.nvfp4_quant(x, per_row=False)
    assert g3.shape == (1,) and g3[0] == g
    assert np.array_equal(sb3, sb)


def test_nvfp4_quant_error_bound_and_invariants():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((16, 256)) * np.exp(rng.uniform(-4, 4, (16, 1)))).astype(np.float32)
    q, sb, g = oracle.nvfp4_quant(x, per_row=True)
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(g, (amax / np.float32(2688)).astype(np.float32))
    d = oracle.nvfp4_dequant(q, sb, g)
    step = np.repeat(oracle.e4m3_decode(sb), 16, axis=1) * g[:, None].astype(np.float64)
    # largest E2M1 gap is 2 (between 4 and 6): error <= 1 scale step, and a
    # little more only when the block scale rounded down and 6 saturated
    assert np.all(np.abs(d - x) <= 1.0 * step * (1 + 1e-6))
    # the block holding the row maximum has scale 448 and a code of +-6 there
    for r in range(x.shape[0]):
        k = int(np.argmax(np.abs(x[r])))
        assert sb[r, k // 16] == 0x7E
        assert abs(oracle.e2m1_decode(q[r, k])) == 6.0


def test_nvfp4_quant_special_rows():
    x = np.zeros((3, 32), dtype=np.float32)
    x[1, 5] = -3.0       # one nonzero element
    x[2, :16] = 1.0      # a second block of zeros next to a full one
    q, sb, g = oracle.nvfp4_quant(x, per_row=True)
    assert g[0] == 0 and np.all(sb[0] == 0) and np.all(oracle.e2m1_decode(q[0]) == 0)
    assert g[1] == np.float32(3.0) / np.float32(2688)
    assert sb[1, 0] == 0x7E and oracle.e2m1_decode(q[1, 5]) == -6.0
    assert sb[1, 1] == 0
    assert np.all(oracle.e2m1_decode(q[2, :16]) == 6.0) and sb[2, 1] == 0


def test_nvfp4_bf16_input_is_widened_exactly():
    rng = np.random.default_rng(2)
    f = rng.standard_normal((4, 64)).astype(np.float32)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    a = oracle.nvfp4_quant(bits)
    b = oracle.nvfp4_quant(oracle.bf16_to_float(bits))
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_e2m1_pack_layout():
    q = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    assert list(oracle.e2m1_pack(q)[0]) == [0x21, 0x43]
    assert np.array_equal(oracle.e2m1_unpack(oracle.e2m1_pack(q)), q)


@pytest.mark.parametrize("M,N,K", [(5, 7, 32), (9, 3, 256)])
def test_nvfp4_gemm_equals_float64_matmul(M, N, K):
    rng = np.random.default_rng(M * 100 + K)
    qa = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    qb = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    sa = rng.integers(0, 0x7F, size=(M, K // 16)).astype(np.uint8)
    sbb = rng.integers(0, 0x7F, size=(N, K // 16)).astype(np.uint8)
    ga = rng.uniform(0.5, 2, M).astype(np.float32)
    gb = np.float32(0.75)
    y, y64 = oracle.nvfp4_gemm(qa, sa, ga, qb, sbb, gb)
    A = oracle.nvfp4_dequant(qa, sa, np.ones(M))
    B = oracle.nvfp4_dequant(qb, sbb, np.ones(N))
    # every product and partial sum is exact in float64 at these sizes
    want = (A @ B.T) * ga.astype(np.float64)[:, None] * np.float64(gb)
    assert np.allclose(y64, want, rtol=1e-15, atol=0)
    assert np.array_equal(y, oracle.bf16_from_double(y64))


def test_nvfp4_gemm_one_block_scale_moves_one_block():
    # doubling one block scale of A doubles exactly that block's contribution
    rng = np.random.default_rng(8)
    M, N, K = 2, 3, 64
    qa = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    qb = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    sa = np.full((M, K // 16), 0x38, dtype=np.uint8)  # 1.0
    sbb = np.full((N, K // 16), 0x38, dtype=np.uint8)
    ga = np.ones(M, dtype=np.float32)
    _, base = oracle.nvfp4_gemm(qa, sa, ga, qb, sbb, 1.0)
    sa2 = sa.copy()
    sa2[1, 2] = 0x40  # 2.0 on row 1, k = 32 .. 47
    _, moved = oracle.nvfp4_gemm(qa, sa2, ga, qb, sbb, 1.0)
    blk = oracle.e2m1_decode(qa[1, 32:48]) @ oracle.e2m1_decode(qb[:, 32:48]).T
    assert np.array_equal(moved[0], base[0])
    assert np.array_equal(moved[1] - base[1], blk)


def test_moe_forward_nvfp4_composes_its_steps():
    rng = np.random.default_rng(21)
    T, H, I, E, k = 6, 64, 32, 3, 2
    x = (rng.standard_normal((T, H)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0, 1, (T, k)).astype(np.float32)

    def weights(N, K):
        qs, ss, gs = [], [], []
        for _ in range(E):
            q, s, g = oracle.nvfp4_quant(rng.standard_normal((N, K)).astype(np.float32),
                                         per_row=False)
            qs.append(q), ss.append(s), gs.append(g[0])
        return np.stack(qs), np.stack(ss), np.array(gs, dtype=np.float32)

    up, dn = weights(I, H), weights(H, I)
    r = oracle.moe_forward_nvfp4(x, ids, w, up, dn)
    # slot (t, j) of the up projection is the plain NVFP4 GEMM of token t
    qx, sx, gx = oracle.nvfp4_quant(x)
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            h, _ = oracle.nvfp4_gemm(qx[t:t + 1], sx[t:t + 1], gx[t:t + 1], up[0][e], up[1][e],
                                     up[2][e])
            assert np.array_equal(r["h"][t * k + j], h[0])
    # the combine is the weighted float64 sum of the slots, rounded once
    o = oracle.bf16_to_float(r["o"]).astype(np.float64).reshape(T, k, H)
    want = oracle.bf16_from_double((o * w.astype(np.float64)[:, :, None]).sum(axis=1))
    assert np.array_equal(r["y"], want)
    # a subset of tokens gives the same rows
    sub = oracle.moe_forward_nvfp4(x, ids, w, up, dn, tokens=[4, 1])
    assert np.array_equal(sub["y"], r["y"][[4, 1]])
