"""Pins of the oracle's routed-expert path: routing bookkeeping against
numpy's stable sort, the combine against exact rationals, and the whole
layer against its degenerate cases (one expert; identical experts)."""
from fractions import Fraction

import numpy as np

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
