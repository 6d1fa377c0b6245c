"""Failure detection on the GPU without a fault: the kernels' bounded
mbarrier wait, run on a barrier that nothing completes, gives up after its
limit, sets the device error word and returns; the host reads (and clears)
KDA_ERR_DEVICE_TIMEOUT and the context keeps working."""
import time

import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W
from parity_util import compare_units

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_reports_and_leaves_the_context_usable(cuda_device):
    assert kda.device_error() == 0
    t0 = time.perf_counter()
    kda.selftest_bounded_wait(50_000_000)  # 50 ms
    code = kda.device_error()
    elapsed = time.perf_counter() - t0
    assert code == 6  # KDA_ERR_DEVICE_TIMEOUT
    assert 0.04 <= elapsed < 5.0
    assert kda.device_error() == 0  # read-and-clear
    # the context still runs the prefill correctly
    inp = W.make_prefill(1, 100, 2, 128, 128, "bf16", -3.0, 1.0, 0.05, seed=60, device=cuda_device)
    o, S = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], None, 64)
    torch.cuda.synchronize()
    compare_units(inp, o, S, [(0, 0), (0, 1)], 1e-2)
    assert kda.device_error() == 0
