"""The allocation-free routed-expert entry point.

metis_moe_fp8_grouped_gemm_noalloc is for callers that cannot allocate device
memory themselves (for instance a host program inside an engine that planned
all GPU memory when it loaded, or a plugin given pointers but no allocator):
it takes no workspace and uses a 16 MiB scratch array built into the library.
These tests call it through the C ABI and compare it with the workspace entry
point, on two calls in a row with different inputs (the shared array keeps
the first call's contents when the second one runs), within the tolerance of
the other parity tests. This file sorts last so that a run stopping at the
first failure has already run every other test; it also passes on its own.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_gemm_token_b200 import synth
from gpu_helpers import assert_close, bf16_dev, bf16_host, dev

pytestmark = pytest.mark.gpu


def _inputs(seed, T, H, I, E, k):
    d = synth.moe(seed=seed, T=T, H=H, I=I, E=E, topk=k, hot=2, load_ratio=2.0)
    up = [oracle.quant_per_channel(d["w_up"][e]) for e in range(E)]
    dn = [oracle.quant_per_channel(d["w_down"][e]) for e in range(E)]
    return dict(
        x=bf16_dev(d["x"]), ids=dev(d["topk_ids"]), w=dev(d["topk_w"]),
        wu=dev(np.stack([u[0] for u in up])), su=dev(np.stack([u[1] for u in up])),
        wd=dev(np.stack([u[0] for u in dn])), sd=dev(np.stack([u[1] for u in dn])),
        T=T, H=H, I=I, E=E, k=k)


def test_noalloc_matches_workspace_entry_point_twice(metis):
    cases = [_inputs(31, 96, 512, 256, 16, 4), _inputs(32, 160, 256, 512, 8, 2)]
    for i, c in enumerate(cases):
        T, H, I, E, k = c["T"], c["H"], c["I"], c["E"], c["k"]
        ws = torch.empty((metis.metis_workspace_size(metis.METIS_OP_MOE, T, I, H, k, E),),
                         dtype=torch.uint8, device="cuda")
        y_ws = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
        y_na = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        metis.metis_moe_fp8_grouped_gemm(c["x"], c["ids"], c["w"], c["wu"], c["su"], c["wd"],
                                         c["sd"], y_ws, ws)
        metis.metis_moe_fp8_grouped_gemm_noalloc(c["x"], c["ids"], c["w"], c["wu"], c["su"],
                                                 c["wd"], c["sd"], y_na)
        assert metis.metis_check_device_status() == 0
        ref = bf16_host(y_ws)
        got = bf16_host(y_na)
        ref64 = (ref.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        assert_close(got, ref64, f"noalloc call {i + 1}")
        # same kernels, same order: the results are also identical bit for bit
        assert np.array_equal(got, ref), f"noalloc call {i + 1} differs in some bits"


def test_noalloc_rejects_problems_beyond_its_scratch(metis):
    T, H, I, E, k = 4096, 2048, 1024, 64, 8   # needs about 296 MiB of scratch
    x = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    w = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    wu = torch.zeros((E, I, H), dtype=torch.uint8, device="cuda")
    wd = torch.zeros((E, H, I), dtype=torch.uint8, device="cuda")
    su = torch.zeros((E, I), dtype=torch.float32, device="cuda")
    sd = torch.zeros((E, H), dtype=torch.float32, device="cuda")
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(metis.MetisError) as ei:
        metis.metis_moe_fp8_grouped_gemm_noalloc(x, ids, w, wu, su, wd, sd, y)
    assert ei.value.code == metis.METIS_ERR_INVALID_ARG
    assert "16 MiB" in str(ei.value)
