"""Decode steps captured in a CUDA graph (the way a serving loop replays them).

pa_decode launches the partition kernel and then the merge kernel with
programmatic dependent launch; pa_decode_mla does the same with the MLA
kernel.  Both are captured on a side stream with caller-owned output and
workspace, and replayed.  Each replay must equal the eager call bitwise, and
the eager call must match the float64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2


def u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def pa():
    import paged_split_kv_attention_b200 as m
    return m


def to_dev(inp, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def assert_close(gpu, ref, what):
    g = gpu.float().cpu().numpy().astype(np.float64)
    bad = np.abs(g - ref) > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), f"{what}: {int(bad.sum())}/{bad.size} outside tolerance"


def capture_and_replay(fn, out, replays=3):
    """fn() writes `out`; eager result, then `replays` graph replays compared with it."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()                                   # first use: attributes, tensor maps, sizes
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(replays):
        out.fill_(3.0)
        g.replay()
        torch.cuda.synchronize()
        assert pa().device_status() == 0
        assert torch.equal(out, eager)
    del g
    return eager


@pytest.fixture(scope="module")
def dev(cuda_device):
    return cuda_device


@pytest.mark.parametrize("name", ["gqa", "mixed"])
def test_gqa_decode_graph(dev, name):
    inp = workloads.make(workloads.get(name, batch=8))
    d = to_dev(inp, dev)
    desc = pa().gqa_desc(d["q"], d["k_cache"], d["block_table"], 0)
    ws = torch.empty(pa().workspace_size(desc), dtype=torch.uint8, device=dev)
    out = torch.empty_like(d["q"])

    def step():
        pa().decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["context_lens"],
                    inp["scale"], out=out, workspace=ws)
    eager = capture_and_replay(step, out)
    ref = oracle.decode(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]),
                        inp["block_table"].numpy(), inp["context_lens"].numpy(), inp["scale"],
                        inp["dtype"])
    assert_close(eager, ref, name)


def test_mla_decode_graph(dev):
    inp = workloads.make(workloads.get("mla", batch=4))
    d = to_dev(inp, dev)
    desc = pa().mla_desc(d["q"], d["latent_cache"], d["block_table"], 512, 0)
    ws = torch.empty(pa().workspace_size(desc), dtype=torch.uint8, device=dev)
    out = torch.empty((4, 128, 512), dtype=d["q"].dtype, device=dev)

    def step():
        pa().decode_mla(d["q"], d["latent_cache"], d["block_table"], d["context_lens"],
                        inp["scale"], out=out, workspace=ws)
    eager = capture_and_replay(step, out)
    b = np.array([0, 3], np.int32)
    pairs = np.array([(bb, h) for bb in b for h in (0, 77, 127)], np.int32)
    ref = oracle.decode_mla(u16(inp["q"]), u16(inp["latent_cache"]), inp["block_table"].numpy(),
                            inp["context_lens"].numpy(), inp["scale"], inp["dtype"],
                            v_dim=inp["v_dim"], pairs=pairs)
    assert_close(eager[pairs[:, 0], pairs[:, 1]], ref, "mla")
