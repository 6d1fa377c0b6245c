"""Several host threads call the library at once (each on its own stream):
the one-time per-device setup is guarded, the error message is per thread,
and every thread gets the same bits as a single-threaded call."""
import threading

import pytest
import torch

import kimi_delta_attention_31_b200 as kda
import kda_workloads as W

pytestmark = pytest.mark.gpu


def test_concurrent_host_threads(cuda_device):
    inp = W.make_prefill(2, 300, 4, 128, 128, "bf16", -3.0, 1.0, 0.05, seed=800, device=cuda_device)
    o_ref, S_ref = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], None, 64)
    torch.cuda.synchronize()
    results, errors = {}, []

    def worker(i):
        try:
            stream = torch.cuda.Stream(cuda_device)
            with torch.cuda.stream(stream):
                for _ in range(3):
                    o, S = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], None, 64)
                # a failing call in this thread leaves its message here only
                with pytest.raises(kda.KDAError):
                    kda.chunk_fwd(inp["q"][..., :96].contiguous(), inp["k"][..., :96].contiguous(),
                                  inp["v"][..., :96].contiguous(), inp["g"][..., :96].contiguous(), inp["beta"],
                                  None, None, 64)
                msg = kda.last_error()
            stream.synchronize()
            results[i] = (o, S, msg)
        except Exception as e:  # noqa: BLE001  (reported below)
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(4)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for o, S, msg in results.values():
        assert torch.equal(o, o_ref) and torch.equal(S, S_ref)
        assert "dk=96" in msg
