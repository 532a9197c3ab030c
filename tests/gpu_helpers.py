"""Helpers shared by the GPU parity tests: numpy <-> device tensors and the
tolerance of the floating-point outputs.

Tolerance (the bar of the workload statement): after FP32 accumulation,
|gpu - ref| <= 1e-2 * (1 + |ref|) element-wise, with ref the oracle's exact
(float64) value. Quantized bytes and scales are compared bit-exactly.
"""
import numpy as np
import torch

RTOL = 1e-2


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_dev(bits):
    """uint16 BF16 bit patterns -> torch.bfloat16 CUDA tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_host(t):
    """torch.bfloat16 tensor -> uint16 numpy bit patterns."""
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_close(gpu_bits, ref64, what=""):
    """GPU BF16 output vs the oracle's exact value: |d| <= 1e-2 (1 + |ref|)."""
    g = bf16_to_f64(gpu_bits)
    r = np.asarray(ref64, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - r)
    bound = RTOL * (1.0 + np.abs(r))
    bad = np.nonzero(err > bound)
    if bad[0].size:
        idx = tuple(b[0] for b in bad)
        raise AssertionError(f"{what}: {bad[0].size} of {g.size} outside tolerance; first at {idx}: "
                             f"gpu={g[idx]} ref={r[idx]}")
    return float((err / (1.0 + np.abs(r))).max()) if err.size else 0.0


def assert_bytes_equal(gpu, ref, what=""):
    gpu = np.asarray(gpu)
    ref = np.asarray(ref)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    bad = np.nonzero(gpu != ref)
    if bad[0].size:
        idx = tuple(b[0] for b in bad)
        raise AssertionError(f"{what}: {bad[0].size} of {gpu.size} differ; first at {idx}: "
                             f"gpu={gpu[idx]!r} ref={ref[idx]!r}")
