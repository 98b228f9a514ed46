"""GPU parity of the sequence-length sweep's largest points against the oracle.

The sweep (bench.py --sweep mha|mqa) runs every length from 512 to 65536 in two
launch configurations: the default split over the whole GPU and one CTA per 8
(sequence, kv head) segments.  At 65536 tokens, both configurations are checked
on sampled heads against the float64 oracle, with the tolerance of the other
parity tests.
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


@pytest.mark.parametrize("kind", ["mha", "mqa"])
def test_longest_sweep_point_both_launches(cuda_device, kind):
    import paged_split_kv_attention_b200 as pa
    w = workloads.scaling(kind, workloads.SWEEP_CTX[-1], 1)
    inp = workloads.make(w)
    d = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    heads = [0, 5, 15]
    pairs = np.array([[0, h] for h in heads], np.int32)
    ref = oracle.decode(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]),
                        inp["block_table"].numpy(), inp["context_lens"].numpy(), inp["scale"],
                        inp["dtype"], pairs=pairs)
    segments = w.batch * w.num_kv_heads
    for parts in (0, -(-segments // 8)):
        out = pa.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["context_lens"],
                        inp["scale"], num_partitions=parts)
        torch.cuda.synchronize()
        assert pa.device_status() == pa.PA_OK
        g = out[0, heads].float().cpu().numpy().astype(np.float64)
        err = np.abs(g - ref)
        assert (err <= ATOL + RTOL * np.abs(ref)).all(), (kind, parts, err.max())
