"""GPU parity of the routed-expert layer, stage by stage, against the oracle.

Integer stages (histogram, offsets, permutation) and quantized bytes/scales
are bit-exact; BF16 stages are within 1e-2 * (1 + |ref|). Each BF16 stage is
checked against the oracle applied to the GPU's own input of that stage, and
the whole layer against the oracle end to end."""
import numpy as np
import pytest
import torch

import oracle
from moe_gemm_token_b200 import synth
from gpu_helpers import assert_bytes_equal, assert_close, bf16_dev, bf16_host, dev

pytestmark = pytest.mark.gpu


def _region(metis, ws, name, shape, dtype, T, k, E, H, I):
    off = metis.metis_moe_workspace_offset(name, T, k, E, H, I)
    nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    return ws[off:off + nbytes].view(dtype).view(*shape)


def run_moe(metis, d):
    T, H, I, E, k = d["T"], d["H"], d["I"], d["E"], d["topk"]
    up = [oracle.quant_per_channel(d["w_up"][e]) for e in range(E)]
    dn = [oracle.quant_per_channel(d["w_down"][e]) for e in range(E)]
    wq_up = np.stack([u[0] for u in up]); s_up = np.stack([u[1] for u in up])
    wq_dn = np.stack([u[0] for u in dn]); s_dn = np.stack([u[1] for u in dn])
    ws_bytes = metis.metis_workspace_size(metis.METIS_OP_MOE, T, I, H, k, E)
    ws = torch.zeros((ws_bytes,), dtype=torch.uint8, device="cuda")
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    metis.metis_moe_fp8_grouped_gemm(bf16_dev(d["x"]), dev(d["topk_ids"]), dev(d["topk_w"]),
                                     dev(wq_up), dev(s_up), dev(wq_dn), dev(s_dn), y, ws)
    assert metis.metis_check_device_status() == 0
    S = T * k
    R = lambda name, shape, dt: _region(metis, ws, name, shape, dt, T, k, E, H, I).cpu().numpy()
    out = dict(
        counts=R("COUNTS", (E,), torch.int32), offsets=R("OFFSETS", (E + 1,), torch.int32),
        s2r=R("SLOT_TO_ROW", (S,), torch.int32), r2s=R("ROW_TO_SLOT", (S,), torch.int32),
        aq=R("AQ", (S, H), torch.uint8), sa=R("SA", (S,), torch.float32),
        h=R("H", (S, I), torch.int16).view(np.uint16), hq=R("HQ", (S, I), torch.uint8),
        sh=R("SH", (S,), torch.float32), o=R("O", (S, H), torch.int16).view(np.uint16),
        y=bf16_host(y), wq_up=wq_up, s_up=s_up, wq_dn=wq_dn, s_dn=s_dn)
    return out


def check_moe(d, g, tokens=None):
    T, k, E = d["T"], d["topk"], d["E"]
    ids = d["topk_ids"]
    # integer stages: bit-exact
    counts, offsets, s2r, r2s = oracle.moe_route(ids, E)
    assert_bytes_equal(g["counts"], counts, "counts")
    assert_bytes_equal(g["offsets"], offsets, "offsets")
    assert_bytes_equal(g["s2r"], s2r, "slot_to_row")
    assert_bytes_equal(g["r2s"], r2s, "row_to_slot")
    # per-token codes of x, written into every row the token was routed to
    xq, sx = oracle.quant_per_token(d["x"])
    tok_of_row = r2s // k
    assert_bytes_equal(g["aq"], xq[tok_of_row], "x codes in expert order")
    assert_bytes_equal(g["sa"].view(np.uint32), sx[tok_of_row].view(np.uint32), "x scales in expert order")
    slots = np.arange(T * k) if tokens is None else \
        (np.asarray(tokens)[:, None] * k + np.arange(k)).reshape(-1)
    rows = s2r[slots]
    exp = ids.reshape(-1)[slots]
    # up-projection on the GPU's gathered operands
    _, h64 = oracle.moe_expert_gemm(g["aq"][rows], g["sa"][rows], g["wq_up"], g["s_up"], exp)
    assert_close(g["h"][rows], h64, "h")
    # re-quantization of the GPU's h: bit-exact
    hq, sh = oracle.quant_per_token(g["h"][rows])
    assert_bytes_equal(g["hq"][rows], hq, "h codes")
    assert_bytes_equal(g["sh"][rows].view(np.uint32), sh.view(np.uint32), "h scales")
    # down-projection on the GPU's codes
    _, o64 = oracle.moe_expert_gemm(g["hq"][rows], g["sh"][rows], g["wq_dn"], g["s_dn"], exp)
    assert_close(g["o"][rows], o64, "o")
    # combine on the GPU's o
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    o_slots = g["o"][rows].reshape(toks.size, k, -1)
    _, y64 = oracle.moe_combine(o_slots, d["topk_w"][toks])
    assert_close(g["y"][toks], y64, "y (combine)")
    # end to end against the oracle alone
    ref = oracle.moe_forward(d["x"], ids, d["topk_w"], g["wq_up"], g["s_up"], g["wq_dn"],
                             g["s_dn"], tokens=toks)
    assert_close(g["y"][toks], ref["y64"], "y (end to end)")


@pytest.mark.parametrize("T,H,I,E,k,seed", [(200, 256, 128, 8, 2, 11), (300, 512, 256, 64, 8, 12),
                                            (37, 128, 272, 5, 3, 13), (1, 64, 32, 4, 4, 14),
                                            (513, 256, 512, 16, 1, 15),
                                            (96, 2048, 256, 16, 4, 18),   # K = 2048: CTA-pair tiles
                                            # pairs, I = 1040: 5 column tiles, the last 16 wide
                                            (150, 1024, 1040, 6, 2, 19)])
def test_moe_parity(metis, T, H, I, E, k, seed):
    d = synth.moe(seed=seed, T=T, H=H, I=I, E=E, topk=k, hot=min(2, E), load_ratio=2.0)
    g = run_moe(metis, d)
    check_moe(d, g)


@pytest.mark.parametrize("T,H,I,E,k,seed", [(300, 256, 128, 16, 9, 42), (1024, 1024, 128, 16, 10, 43)])
def test_moe_parity_more_than_eight_experts_per_token(metis, T, H, I, E, k, seed):
    """More than 8 experts per token take the combine's general loop (the
    row indices read inside the sum); with 1024 tokens x 128 column groups
    every thread of the persistent grid walks several items."""
    d = synth.moe(seed=seed, T=T, H=H, I=I, E=E, topk=k, hot=2, load_ratio=2.0)
    g = run_moe(metis, d)
    check_moe(d, g)


@pytest.mark.parametrize("T,E,k,seed", [(64, 320, 4, 40), (4096, 160, 8, 41)])
def test_moe_routing_without_the_fused_scan(metis, T, E, k, seed):
    """Routing tables too large for the fused prefix-sum and rank kernel (more
    than 256 experts; more than 16384 per-chunk counts: 128 chunks x 160
    experts) take the single-block scan and the rank kernel; every stage
    still matches the oracle."""
    d = synth.moe(seed=seed, T=T, H=128, I=64, E=E, topk=k, hot=4, load_ratio=2.0)
    g = run_moe(metis, d)
    check_moe(d, g)


def test_moe_empty_experts(metis):
    """Experts that receive no token produce no tiles; the others are unaffected."""
    d = synth.moe(seed=16, T=64, H=128, I=64, E=16, topk=2, hot=0, load_ratio=1.0)
    ids = d["topk_ids"]
    ids[:, 0] = 3
    ids[:, 1] = 9  # only experts 3 and 9 are used
    d["topk_ids"] = ids
    g = run_moe(metis, d)
    assert g["counts"].tolist().count(0) == 14
    check_moe(d, g)


def test_moe_deterministic(metis):
    d = synth.moe(seed=17, T=256, H=256, I=128, E=8, topk=2, hot=2, load_ratio=2.0)
    a = run_moe(metis, d)
    b = run_moe(metis, d)
    for key in ("y", "h", "o", "s2r"):
        assert np.array_equal(a[key], b[key]), key


# ---------------------------------------------------------------- router top-k

def _route_gpu(metis, logits32, k, bias32=None):
    T, E = logits32.shape
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    metis.metis_moe_route_topk(dev(logits32), ids, w, bias=None if bias32 is None else dev(bias32))
    assert metis.metis_check_device_status() == 0
    return ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T,E,k,seed,with_bias", [(4096, 64, 8, 20, False), (4096, 64, 8, 21, True),
                                                  (333, 100, 4, 22, True), (64, 7, 7, 23, False),
                                                  (50, 1024, 32, 24, True), (257, 192, 4, 25, True)])
def test_route_topk_parity(metis, T, E, k, seed, with_bias):
    """Ids bit-exact against the oracle (the same binary32 scores decide);
    weights within 1e-5 (FP32 softmax against float64)."""
    rng = np.random.default_rng(seed)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    b = (rng.standard_normal(E) * 0.5).astype(np.float32) if with_bias else None
    ids, w = _route_gpu(metis, lg, k, b)
    ids_r, w_r = oracle.route_topk(lg, k, b)
    assert_bytes_equal(ids, ids_r, "router ids")
    assert np.max(np.abs(w.astype(np.float64) - w_r)) <= 1e-5


def test_route_topk_ties_and_infinities(metis):
    """Integer logits (ties everywhere) and -inf logits: the lower expert
    index wins ties; -inf experts are chosen last."""
    rng = np.random.default_rng(26)
    lg = rng.integers(-2, 3, (512, 40)).astype(np.float32)
    lg[:, 5] = -np.inf
    lg[::7, :] = 1.0  # whole rows tied
    b = (rng.integers(-1, 2, 40) * 0.5).astype(np.float32)
    cases = [(lg, 1, None), (lg, 8, None), (lg, 8, b), (lg, 32, b),
             (np.ascontiguousarray(lg[:, :20]), 20, b[:20].copy())]  # all chosen: -inf last
    for lgc, k, bias in cases:
        ids, w = _route_gpu(metis, lgc, k, bias)
        ids_r, w_r = oracle.route_topk(lgc, k, bias)
        assert_bytes_equal(ids, ids_r, f"router ids k={k}")
        assert np.max(np.abs(w.astype(np.float64) - w_r)) <= 1e-5


def test_route_topk_feeds_the_layer(metis):
    """The routed-expert layer fed by the GPU router equals the oracle layer
    fed by the oracle router (same ids; weights within 1e-5)."""
    d = synth.moe(seed=27, T=192, H=256, I=128, E=16, topk=4, hot=2, load_ratio=2.0)
    lg = d["logits"].astype(np.float32)
    ids, w = _route_gpu(metis, lg, 4)
    ids_r, w_r = oracle.route_topk(lg, 4)
    assert_bytes_equal(ids, ids_r, "router ids")
    d["topk_ids"], d["topk_w"] = ids, w
    g = run_moe(metis, d)
    ref = oracle.moe_forward(d["x"], ids_r, w_r.astype(np.float32), g["wq_up"], g["s_up"], g["wq_dn"],
                             g["s_dn"])
    assert_close(g["y"], ref["y64"], "layer fed by the GPU router")


def test_moe_out_of_range_ids_are_dropped_and_reported(metis):
    """Routing ids stay on the GPU, so the host cannot check them: an id
    outside [0, E) drops that slot (its SLOT_TO_ROW entry is -1 and it adds
    nothing to y), sets the sticky status word (reported as
    METIS_ERR_INVALID_ARG) and leaves every other slot as the oracle computes
    it. The reference: the same layer with the bad slot's weight set to 0 (and
    any valid id in its place, which only moves rows within an expert)."""
    d = synth.moe(seed=28, T=128, H=256, I=128, E=8, topk=2, hot=2, load_ratio=2.0)
    E = d["E"]
    ids = d["topk_ids"].copy()
    bad = [(5, 1, E), (77, 0, E + 3), (100, 1, -1)]
    for t, j, v in bad:
        ids[t, j] = v
    d_bad = dict(d, topk_ids=ids)
    metis.metis_check_device_status()  # start clean
    T, H, I, k = d["T"], d["H"], d["I"], d["topk"]
    up = [oracle.quant_per_channel(d["w_up"][e]) for e in range(E)]
    dn = [oracle.quant_per_channel(d["w_down"][e]) for e in range(E)]
    wq_up = np.stack([u[0] for u in up]); s_up = np.stack([u[1] for u in up])
    wq_dn = np.stack([u[0] for u in dn]); s_dn = np.stack([u[1] for u in dn])
    ws = torch.zeros((metis.metis_workspace_size(metis.METIS_OP_MOE, T, I, H, k, E),),
                     dtype=torch.uint8, device="cuda")
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    metis.metis_moe_fp8_grouped_gemm(bf16_dev(d_bad["x"]), dev(ids), dev(d["topk_w"]), dev(wq_up),
                                     dev(s_up), dev(wq_dn), dev(s_dn), y, ws)
    assert metis.metis_check_device_status(clear=False) == metis.METIS_ERR_INVALID_ARG
    assert metis.metis_check_device_status(clear=True) == metis.METIS_ERR_INVALID_ARG
    assert metis.metis_check_device_status() == 0  # cleared
    s2r = _region(metis, ws, "SLOT_TO_ROW", (T * k,), torch.int32, T, k, E, H, I).cpu().numpy()
    for t, j, _ in bad:
        assert s2r[t * k + j] == -1
    counts = _region(metis, ws, "COUNTS", (E,), torch.int32, T, k, E, H, I).cpu().numpy()
    assert counts.sum() == T * k - len(bad)
    ids_ref = ids.copy()
    w_ref = d["topk_w"].copy()
    for t, j, _ in bad:
        ids_ref[t, j] = (ids[t, 1 - j] + 1) % E  # any valid expert other than the token's other one
        w_ref[t, j] = 0.0
    ref = oracle.moe_forward(d["x"], ids_ref, w_ref, wq_up, s_up, wq_dn, s_dn)
    assert_close(bf16_host(y), ref["y64"], "y with dropped slots")
