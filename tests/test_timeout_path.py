"""GPU tests of the kernels' timeout path, with no fault and no hang.

Every mbarrier wait in the kernels is bounded (about one second).  The test hook
pa_test_inject_stall sets a flag in device memory; while it is set, one warp of
each partition pass waits on a barrier that nothing completes, before it issues
any copy.  The wait must give up, record PA_ERR_TIMEOUT in the device status word
and let the launch finish, and the CUDA context must stay usable: the next call,
with the hook off, returns the same output as before.

The single-pass merge (pa_decode_fused) keeps arrival counters in the workspace,
tagged with a per-call epoch that a captured graph reuses on every replay.  A
piece that timed out still counts itself in, so a replay after a timed-out
replay starts from clean counters and merges correctly.
"""
import time

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def pa():
    import paged_split_kv_attention_b200 as m
    return m


def to_dev(inp, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def stalled(call):
    """Run call() with the hook on; returns the status word and the elapsed time."""
    pa().inject_stall_for_testing(True)
    try:
        t0 = time.time()
        call()
        status = pa().device_status()
        elapsed = time.time() - t0
    finally:
        pa().inject_stall_for_testing(False)
    return status, elapsed


def test_stalled_wait_reports_timeout_and_context_survives(cuda_device):
    inp = workloads.make(workloads.get("gqa", batch=4))
    d = to_dev(inp, cuda_device)

    def call():
        return pa().decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"],
                           d["context_lens"], inp["scale"])

    ref = call()
    assert pa().device_status() == pa().PA_OK
    status, elapsed = stalled(call)
    assert status == pa().PA_ERR_TIMEOUT, pa().status_string(status)
    assert elapsed < 30.0
    out = call()
    assert pa().device_status() == pa().PA_OK
    assert torch.equal(out, ref)


def test_mla_stalled_wait_reports_timeout_and_context_survives(cuda_device):
    inp = workloads.make(workloads.get("mla", batch=4))
    d = to_dev(inp, cuda_device)

    def call():
        return pa().decode_mla(d["q"], d["latent_cache"], d["block_table"], d["context_lens"],
                               inp["scale"], v_dim=inp["v_dim"])

    ref = call()
    assert pa().device_status() == pa().PA_OK
    status, elapsed = stalled(call)
    assert status == pa().PA_ERR_TIMEOUT, pa().status_string(status)
    assert elapsed < 30.0
    out = call()
    assert pa().device_status() == pa().PA_OK
    assert torch.equal(out, ref)


def test_fused_graph_replays_cleanly_after_a_timeout(cuda_device):
    # 40 partitions x 8 warps over 8 sequences: every segment is split, so the
    # stalled warp (warp 0 of CTA 0) shares its segment with other pieces
    inp = workloads.make(workloads.get("gqa", batch=8))
    d = to_dev(inp, cuda_device)
    desc = pa().gqa_desc(d["q"], d["k_cache"], d["block_table"], 40)
    ws = torch.empty(pa().workspace_size(desc), dtype=torch.uint8, device=cuda_device)
    out = torch.empty_like(d["q"])

    def step():
        pa().decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["context_lens"],
                    inp["scale"], out=out, workspace=ws, num_partitions=40, passes="fused")

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert pa().device_status() == pa().PA_OK
    eager = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    try:
        g.replay()
        torch.cuda.synchronize()
        assert pa().device_status() == pa().PA_OK
        assert torch.equal(out, eager)
        status, _ = stalled(lambda: g.replay())
        assert status == pa().PA_ERR_TIMEOUT, pa().status_string(status)
        for _ in range(2):
            out.fill_(3.0)
            g.replay()
            torch.cuda.synchronize()
            assert pa().device_status() == pa().PA_OK
            assert torch.equal(out, eager)
    finally:
        del g
