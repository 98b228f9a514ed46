"""GPU test of the kernels' timeout path, with no fault and no hang.

Every mbarrier wait in the kernels is bounded (about one second).  The test hook
pa_test_inject_stall makes one warp of the GQA partition pass wait on a barrier
that nothing completes, before it issues any copy; the wait must give up,
record PA_ERR_TIMEOUT in the device status word and let the launch finish, and
the CUDA context must stay usable: the next call, with the hook off, returns
the same output as before.
"""
import time

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def test_stalled_wait_reports_timeout_and_context_survives(cuda_device):
    import paged_split_kv_attention_b200 as pa
    inp = workloads.make(workloads.get("gqa", batch=4))
    d = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}

    def call():
        return pa.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["context_lens"],
                         inp["scale"])

    ref = call()
    assert pa.device_status() == pa.PA_OK
    pa.inject_stall_for_testing(True)
    try:
        t0 = time.time()
        call()
        status = pa.device_status()
        elapsed = time.time() - t0
    finally:
        pa.inject_stall_for_testing(False)
    assert status == pa.PA_ERR_TIMEOUT, pa.status_string(status)
    assert elapsed < 30.0
    out = call()
    assert pa.device_status() == pa.PA_OK
    assert torch.equal(out, ref)
