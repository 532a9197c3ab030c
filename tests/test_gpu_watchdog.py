"""Failure detection on the GPU without a GPU fault: a bounded wait that
nothing satisfies runs out, the kernel returns, the host reads
METIS_ERR_TIMEOUT from the sticky status word, and the context keeps
working."""
import numpy as np
import pytest
import torch

import oracle
from moe_gemm_token_b200 import synth
from gpu_helpers import assert_bytes_equal, bf16_dev

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported(metis):
    assert metis.metis_check_device_status() == 0
    metis.metis_watchdog_selftest(2_000_000)  # 2 ms
    assert metis.metis_check_device_status(clear=True) == metis.METIS_ERR_TIMEOUT
    assert metis.metis_check_device_status() == 0  # cleared
    # the context still computes correctly
    d = synth.tiny_linear()
    xq = torch.empty((16, 256), dtype=torch.uint8, device="cuda")
    s = torch.empty((16,), dtype=torch.float32, device="cuda")
    metis.metis_quant_fp8_per_token(bf16_dev(d["x"]), xq, s)
    assert metis.metis_check_device_status() == 0
    xq_r, s_r = oracle.quant_per_token(d["x"])
    assert_bytes_equal(xq.cpu().numpy(), xq_r, "codes after a timeout")
    assert_bytes_equal(s.cpu().numpy().view(np.uint32), s_r.view(np.uint32), "scales after a timeout")


def test_status_is_sticky_until_cleared(metis):
    metis.metis_watchdog_selftest(1_000_000)
    assert metis.metis_check_device_status(clear=False) == metis.METIS_ERR_TIMEOUT
    assert metis.metis_check_device_status(clear=True) == metis.METIS_ERR_TIMEOUT
    assert metis.metis_check_device_status() == 0
