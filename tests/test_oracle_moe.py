"""Pins of the oracle's routed-expert path: routing bookkeeping against
numpy's stable sort, the combine against exact rationals, the whole layer
against its degenerate cases (one expert; identical experts), and the router
top-k against an independent sort, the plain softmax and its invariants."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from moe_gemm_token_b200 import synth


def _small_moe(seed=7, T=40, H=64, I=32, E=6, topk=3):
    d = synth.moe(seed=seed, T=T, H=H, I=I, E=E, topk=topk, hot=2, load_ratio=1.5)
    up = [oracle.quant_per_channel(d["w_up"][e]) for e in range(E)]
    dn = [oracle.quant_per_channel(d["w_down"][e]) for e in range(E)]
    d["wq_up"] = np.stack([u[0] for u in up]); d["s_up"] = np.stack([u[1] for u in up])
    d["wq_down"] = np.stack([u[0] for u in dn]); d["s_down"] = np.stack([u[1] for u in dn])
    return d


def test_route_matches_stable_argsort():
    d = synth.moe(seed=3, T=512, H=8, I=8, E=64, topk=8, with_weights=False)
    ids = d["topk_ids"]
    counts, offsets, s2r, r2s = oracle.moe_route(ids, 64)
    flat = ids.reshape(-1)
    assert counts.sum() == flat.size
    assert np.array_equal(counts, np.bincount(flat, minlength=64))
    assert offsets[0] == 0 and np.all(np.diff(offsets) == counts)
    order = np.argsort(flat, kind="stable")   # rows -> slots, stable by expert
    assert np.array_equal(r2s, order)
    assert np.array_equal(s2r[order], np.arange(flat.size))
    # bijection and per-expert contiguity
    assert np.array_equal(np.sort(s2r), np.arange(flat.size))
    for e in range(64):
        rows = s2r[flat == e]
        assert np.all((rows >= offsets[e]) & (rows < offsets[e + 1]))
        assert np.all(np.diff(rows) == 1)


def test_route_workload_histogram_is_skewed():
    d = synth.moe(with_weights=False)
    counts, _, _, _ = oracle.moe_route(d["topk_ids"], d["E"])
    hot = counts[d["hot_experts"]].mean()
    assert abs(hot / (d["T"] * d["topk"] / d["E"]) - 3.0) < 0.02


def test_combine_matches_exact_rationals():
    rng = np.random.default_rng(0)
    T, k, H = 5, 4, 7
    o = synth.f32_to_bf16_bits(rng.standard_normal((T, k, H)))
    w = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    y, _ = oracle.moe_combine(o, w)
    of = synth.bf16_bits_to_f32(o)
    for t in range(T):
        for n in range(H):
            exact = sum(Fraction(float(w[t, j])) * Fraction(float(of[t, j, n])) for j in range(k))
            got = float(synth.bf16_bits_to_f32(y[t, n]))
            # nearest BF16 to the exact value (the float64 sum of 4 terms of
            # 8+24 significant bits is exact here)
            lo = Fraction(got)
            step = Fraction(abs(got)) * Fraction(1, 128) if got else Fraction(1, 2 ** 133)
            assert abs(lo - exact) <= step / 2


def test_single_expert_topk1_is_dense_chain():
    d = _small_moe(E=1, topk=1)
    r = oracle.moe_forward(d["x"], d["topk_ids"], np.ones_like(d["topk_w"]),
                           d["wq_up"], d["s_up"], d["wq_down"], d["s_down"])
    h, _, _, _ = oracle.linear_w8a8(d["x"], d["wq_up"][0], d["s_up"][0])
    y, _, _, _ = oracle.linear_w8a8(h, d["wq_down"][0], d["s_down"][0])
    assert np.array_equal(r["h"], h)
    assert np.array_equal(r["y"], y)


def test_identical_experts_equal_weights_is_dense_chain():
    d = _small_moe(E=4, topk=4)
    for key in ("wq_up", "s_up", "wq_down", "s_down"):
        d[key][:] = d[key][0]
    w = np.full_like(d["topk_w"], 0.25)
    r = oracle.moe_forward(d["x"], d["topk_ids"], w, d["wq_up"], d["s_up"], d["wq_down"],
                           d["s_down"])
    h, _, _, _ = oracle.linear_w8a8(d["x"], d["wq_up"][0], d["s_up"][0])
    y, _, _, _ = oracle.linear_w8a8(h, d["wq_down"][0], d["s_down"][0])
    assert np.array_equal(r["y"], y)


def test_token_subset_matches_full_run():
    d = _small_moe()
    full = oracle.moe_forward(d["x"], d["topk_ids"], d["topk_w"], d["wq_up"], d["s_up"],
                              d["wq_down"], d["s_down"])
    toks = np.array([3, 0, 39, 17])
    sub = oracle.moe_forward(d["x"], d["topk_ids"], d["topk_w"], d["wq_up"], d["s_up"],
                             d["wq_down"], d["s_down"], tokens=toks)
    assert np.array_equal(sub["y"], full["y"][toks])
    k = d["topk"]
    slots = (toks[:, None] * k + np.arange(k)).reshape(-1)
    assert np.array_equal(sub["h"], full["h"][slots])


def test_expert_gemm_uses_each_slots_own_expert():
    """Swapping two experts' weights must change exactly the slots routed to them."""
    d = _small_moe()
    base = oracle.moe_forward(d["x"], d["topk_ids"], d["topk_w"], d["wq_up"], d["s_up"],
                              d["wq_down"], d["s_down"])
    wq = d["wq_up"].copy(); s = d["s_up"].copy()
    wq[[0, 1]] = wq[[1, 0]]; s[[0, 1]] = s[[1, 0]]
    sw = oracle.moe_forward(d["x"], d["topk_ids"], d["topk_w"], wq, s, d["wq_down"],
                            d["s_down"])
    exp = d["topk_ids"].reshape(-1)
    changed = np.any(base["h"] != sw["h"], axis=1)
    assert np.array_equal(changed, np.isin(exp, [0, 1]))


# ---------------------------------------------------------------- router top-k

def _route_reference(logits32, k, bias32=None):
    """Independent restatement: sort by (-score, expert) with the score formed
    by numpy binary32 addition; softmax over the chosen unbiased logits."""
    T, E = logits32.shape
    score = logits32 if bias32 is None else (logits32 + bias32[None, :]).astype(np.float32)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(score[t, e]), e))[:k]
        ids[t] = order
        z = logits32[t, order].astype(np.float64)
        p = np.exp(z - z.max())
        w[t] = p / p.sum()
    return ids, w


def test_route_topk_all_experts_is_the_softmax():
    """k = E: every expert chosen in descending order; the weights are the
    plain softmax of the logits (closed form)."""
    rng = np.random.default_rng(40)
    lg = rng.standard_normal((50, 12)).astype(np.float32)
    ids, w = oracle.route_topk(lg, 12)
    order = np.argsort(-lg.astype(np.float64), axis=1, kind="stable")
    assert np.array_equal(ids, order)
    z = lg.astype(np.float64)
    soft = np.exp(z - z.max(axis=1, keepdims=True))
    soft /= soft.sum(axis=1, keepdims=True)
    assert np.allclose(w, np.take_along_axis(soft, order, axis=1), rtol=1e-13, atol=0)


def test_route_topk_one_expert_gets_weight_one():
    rng = np.random.default_rng(41)
    lg = rng.integers(-3, 4, (200, 16)).astype(np.float32)  # many ties
    ids, w = oracle.route_topk(lg, 1)
    assert np.array_equal(ids[:, 0], np.argmax(lg, axis=1))  # first maximum = lower index
    assert np.all(w == 1.0)


@pytest.mark.parametrize("seed,T,E,k,with_bias", [(42, 64, 6, 3, False), (43, 64, 9, 4, True),
                                                  (44, 32, 16, 8, True), (45, 16, 5, 5, True)])
def test_route_topk_matches_an_independent_sort(seed, T, E, k, with_bias):
    """Small-integer logits and biases force ties; halves make binary32 sums
    exact or rounded. Ids must match a plain sort by (-score, expert)."""
    rng = np.random.default_rng(seed)
    lg = (rng.integers(-4, 5, (T, E)) * 0.5).astype(np.float32)
    lg[:, 0] = lg[:, 1]  # guaranteed ties
    b = (rng.integers(-2, 3, E) * 0.25).astype(np.float32) if with_bias else None
    ids, w = oracle.route_topk(lg, k, b)
    ids_r, w_r = _route_reference(lg, k, b)
    assert np.array_equal(ids, ids_r)
    assert np.allclose(w, w_r, rtol=1e-14, atol=0)


def test_route_topk_bias_decides_the_choice_not_the_weights():
    lg = np.array([[3.0, 2.0, 1.0, 0.5]], np.float32)
    ids, w = oracle.route_topk(lg, 2)
    assert ids.tolist() == [[0, 1]]
    bias = np.array([0.0, 0.0, 5.0, 0.0], np.float32)  # expert 2 overtakes both
    ids_b, w_b = oracle.route_topk(lg, 2, bias)
    assert ids_b.tolist() == [[2, 0]]
    z = np.array([1.0, 3.0])  # unbiased logits of experts 2 and 0
    assert np.allclose(w_b[0], np.exp(z - 3.0) / np.exp(z - 3.0).sum(), rtol=1e-15)
    # a bias that keeps the choice leaves the weights unchanged
    ids_c, w_c = oracle.route_topk(lg, 2, np.array([0.1, 0.1, 0.0, 0.0], np.float32))
    assert ids_c.tolist() == [[0, 1]] and np.array_equal(w_c, w)


def test_route_topk_invariants():
    rng = np.random.default_rng(46)
    lg = rng.standard_normal((300, 64)).astype(np.float32)
    b = (rng.standard_normal(64) * 0.3).astype(np.float32)
    ids, w = oracle.route_topk(lg, 8, b)
    score = lg + b
    for t in range(300):
        assert len(set(ids[t].tolist())) == 8
        chosen = score[t, ids[t]]
        assert np.all(np.diff(chosen) <= 0)  # descending
        others = np.delete(score[t], ids[t])
        assert chosen.min() >= others.max()
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-12)


# ------------------------------------------------------------ shared expert

def _bf16(a):
    return (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_gemm_bf16_equals_float64_matmul():
    rng = np.random.default_rng(31)
    x = _bf16(rng.standard_normal((7, 96)))
    w = _bf16(rng.standard_normal((5, 96)) * 0.05)
    y, y64 = oracle.gemm_bf16(x, w)
    # BF16 products are exact in float64 and these sums stay exact
    want = oracle.bf16_to_float(x).astype(np.float64) @ oracle.bf16_to_float(w).astype(np.float64).T
    assert np.array_equal(y64, want)
    assert np.array_equal(y, oracle.bf16_from_double(want))
    y2, _ = oracle.gemm_bf16(x, w, rows=[4, 1])
    assert np.array_equal(y2, y[[4, 1]])


def test_shared_combine_reduces_to_the_routed_combine_and_to_the_shared_output():
    rng = np.random.default_rng(32)
    T, k, H = 6, 3, 40
    o = _bf16(rng.standard_normal((T, k, H)))
    w = rng.uniform(0, 1, (T, k)).astype(np.float32)
    s = _bf16(rng.standard_normal((T, H)))
    zero = np.zeros((T, H), np.uint16)
    # no shared output: the routed combine
    assert np.array_equal(oracle.shared_combine(zero, o, w)[0], oracle.moe_combine(o, w)[0])
    # no routed weight: the shared output itself, unchanged
    assert np.array_equal(oracle.shared_combine(s, o, np.zeros_like(w))[0], s)
    # the sum, rounded once
    want = oracle.bf16_to_float(s).astype(np.float64) + \
        (oracle.bf16_to_float(o).astype(np.float64) * w.astype(np.float64)[:, :, None]).sum(axis=1)
    y, y64 = oracle.shared_combine(s, o, w)
    assert np.allclose(y64, want, rtol=1e-15, atol=0)
    assert np.array_equal(y, oracle.bf16_from_double(y64))


def test_shared_expert_is_two_rounded_gemms():
    rng = np.random.default_rng(33)
    x = _bf16(rng.standard_normal((4, 64)))
    wu = _bf16(rng.standard_normal((32, 64)) * 0.1)
    wd = _bf16(rng.standard_normal((64, 32)) * 0.1)
    h, s, s64 = oracle.shared_expert(x, wu, wd)
    assert np.array_equal(h, oracle.gemm_bf16(x, wu)[0])
    assert np.array_equal(s, oracle.gemm_bf16(h, wd)[0])
    _, s_sub, _ = oracle.shared_expert(x, wu, wd, tokens=[3, 0])
    assert np.array_equal(s_sub, s[[3, 0]])
