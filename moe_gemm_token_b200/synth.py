"""Seeded synthetic inputs for the FP8 linear-layer workloads.

This module holds no arithmetic of the method itself (no FP8 codec, no
scaling, no GEMM): it only draws numbers. Both the CUDA path and the CPU
oracle read the same arrays from it. BF16 tensors are returned as ``uint16``
bit patterns, rounded from float32 to nearest-even.

Workloads (shapes and value distributions of the pages' setting: FP8 linear
layers of a Mamba-2/attention MoE model, prompt reading, decode and routed
experts):

* ``tiny_linear``   M=16, K=256, N=512; 4 outlier channels x20, row 7 all zero.
* ``prefill_chain`` 4096 tokens, 2048 -> 6144 -> 2048; 1% outlier channels x30.
* ``decode``        M in {1,2,4,8}, K=4096, N=14336.
* ``moe``           4096 tokens, hidden 2048, 64 experts, top-8, latent 1024;
                    4 hot experts with 3x the mean load.
* ``large_m``       M in {8192,16384}, K=N in {4096,8192}; per-token magnitude
                    10**U(-2,2).
"""
import numpy as np


def f32_to_bf16_bits(a):
    """float32 -> BF16 bit patterns, round to nearest-even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(h):
    """Exact widening of BF16 bit patterns to float32."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal(rng, shape, std=1.0):
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def linear(seed, M, K, N, outlier_channels=0, outlier_scale=1.0, zero_rows=(),
           row_magnitude_log10=None, w_std=0.02):
    """Generic linear-layer input: x ~ N(0,1) [M,K] as BF16 and w ~ N(0, w_std)
    [N,K] as float32.

    ``outlier_channels`` seeded channel indices are multiplied by
    ``outlier_scale``; ``zero_rows`` are set to zero; ``row_magnitude_log10``
    = (lo, hi) multiplies each row by 10**U(lo, hi)."""
    rng = np.random.default_rng(seed)
    x = _normal(rng, (M, K))
    ch = np.sort(rng.choice(K, size=outlier_channels, replace=False)) if outlier_channels else \
        np.zeros((0,), dtype=np.int64)
    if ch.size:
        x[:, ch] *= np.float32(outlier_scale)
    if row_magnitude_log10 is not None:
        lo, hi = row_magnitude_log10
        mag = np.power(10.0, rng.uniform(lo, hi, size=(M, 1))).astype(np.float32)
        x *= mag
    for r in zero_rows:
        if 0 <= r < M:
            x[r, :] = 0.0
    w = _normal(rng, (N, K), std=w_std)
    return dict(x=f32_to_bf16_bits(x), w=w, outlier_channels=ch, M=M, K=K, N=N, seed=seed)


def tiny_linear(seed=0):
    """M=16, K=256, N=512; 4 outlier channels x20; row 7 all zero."""
    return linear(seed, 16, 256, 512, outlier_channels=4, outlier_scale=20.0, zero_rows=(7,))


def prefill_chain(seed=1, M=4096, K=2048, N=6144):
    """Two chained linear layers K -> N -> K over M tokens; 1% of the input
    channels are outliers x30; no activation between the layers."""
    rng = np.random.default_rng(seed)
    x = _normal(rng, (M, K))
    n_out = max(1, int(round(0.01 * K)))
    ch = np.sort(rng.choice(K, size=n_out, replace=False))
    x[:, ch] *= np.float32(30.0)
    w1 = _normal(rng, (N, K), std=0.02)
    w2 = _normal(rng, (K, N), std=0.02)
    return dict(x=f32_to_bf16_bits(x), w1=w1, w2=w2, outlier_channels=ch, M=M, K=K, N=N,
                seed=seed)


def decode(seed=2, M=8, K=4096, N=14336):
    """Decode-shaped weight-only input: x ~ N(0,1) [M,K] BF16, w ~ N(0,0.02)."""
    rng = np.random.default_rng(seed)
    x = _normal(rng, (8, K))[:M]
    w = _normal(rng, (N, K), std=0.02)
    return dict(x=f32_to_bf16_bits(x), w=w, M=M, K=K, N=N, seed=seed)


def large_m(seed=4, M=8192, K=4096, N=None):
    """Square-ish sweep input; each token scaled by 10**U(-2,2)."""
    N = K if N is None else N
    return linear(seed, M, K, N, row_magnitude_log10=(-2.0, 2.0))


def _topk_route(logits, topk):
    """Softmax over experts in float64, top-k with ties to the lower index,
    weights renormalised over the chosen k. Returns (ids int32, w float32)."""
    z = logits.astype(np.float64)
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    order = np.argsort(-p, axis=1, kind="stable")[:, :topk]
    pk = np.take_along_axis(p, order, axis=1)
    w = (pk / pk.sum(axis=1, keepdims=True)).astype(np.float32)
    return order.astype(np.int32), w


def moe(seed=3, T=4096, H=2048, I=1024, E=64, topk=8, hot=4, load_ratio=3.0,
        with_weights=True):
    """Routed-expert workload. Router logits ~ N(0,1) [T,E]; ``hot`` seeded
    experts get a bias beta, found by bisection so their mean load is
    ``load_ratio`` x the overall mean (T*topk/E). Expert weights
    w_up [E,I,H] and w_down [E,H,I] ~ N(0,0.02) float32."""
    rng = np.random.default_rng(seed)
    x = _normal(rng, (T, H))
    logits = rng.standard_normal(size=(T, E))
    hot_experts = np.sort(rng.choice(E, size=min(hot, E), replace=False))
    target = load_ratio * T * topk / E

    def hot_load(beta):
        lg = logits.copy()
        lg[:, hot_experts] += beta
        ids, _ = _topk_route(lg, topk)
        return np.bincount(ids.reshape(-1), minlength=E)[hot_experts].mean()

    beta = 0.0
    if hot and load_ratio > 1.0 and E > topk:
        lo, hi = 0.0, 8.0
        for _ in range(40):
            mid = 0.5 * (lo + hi)
            if hot_load(mid) >= target:
                hi = mid
            else:
                lo = mid
        beta = hi
    lg = logits.copy()
    lg[:, hot_experts] += beta
    ids, w = _topk_route(lg, topk)
    out = dict(x=f32_to_bf16_bits(x), logits=lg, topk_ids=ids, topk_w=w, beta=beta,
               hot_experts=hot_experts, T=T, H=H, I=I, E=E, topk=topk, seed=seed,
               histogram=np.bincount(ids.reshape(-1), minlength=E))
    if with_weights:
        out["w_up"] = _normal(rng, (E, I, H), std=0.02)
        out["w_down"] = _normal(rng, (E, H, I), std=0.02)
    return out
