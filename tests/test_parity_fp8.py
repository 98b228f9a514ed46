"""GPU parity of the float8 (E4M3) KV-cache decode against the float64 oracle.

The cache holds E4M3 codes with one key scale and one value scale per tensor;
the oracle decodes the codes exactly and applies the scales in float64.  Same
tolerance as the 16-bit parity tests: |gpu - oracle| <= 2e-3 + 1e-2 |oracle|.
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


def kv8(B, Hq, Hkv, bs, ctx, dtype="bf16", seed=0, pool="factor:1.5"):
    return workloads.GQAWorkload("t", B, Hq, Hkv, 128, dtype, bs,
                                 "fixed:" + ",".join(str(c) for c in ctx), pool, seed,
                                 kv_dtype="e4m3")


def ref_of(inp, k_scale=None, v_scale=None, pairs=None):
    return oracle.decode_kv8(u16(inp["q"]), inp["k_cache"].numpy(), inp["v_cache"].numpy(),
                             inp["k_scale"] if k_scale is None else k_scale,
                             inp["v_scale"] if v_scale is None else v_scale,
                             inp["block_table"].numpy(), inp["context_lens"].numpy(),
                             inp["scale"], inp["dtype"], pairs=pairs)


def run(d, inp, k_scale=None, v_scale=None, **kw):
    out = pa().decode_kv8(d["q"], d["k_cache"], d["v_cache"], d["block_table"],
                          d["context_lens"], inp["scale"],
                          inp["k_scale"] if k_scale is None else k_scale,
                          inp["v_scale"] if v_scale is None else v_scale, **kw)
    torch.cuda.synchronize()
    st = pa().device_status()
    assert st == 0, pa().status_string(st)
    return out


def assert_close(gpu, ref, what=""):
    g = gpu.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), (f"{what}: {int(bad.sum())}/{bad.size} outside tolerance, "
                           f"max abs {err.max():.3e}")
    assert np.isfinite(g).all()


def to_dev(inp, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


@pytest.mark.parametrize("G", [1, 4, 8, 16])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_group_sizes_and_query_types(cuda_device, G, dtype):
    inp = workloads.make(kv8(3, 2 * G, 2, 16, (1, 77, 300), dtype=dtype, seed=G))
    ref = ref_of(inp)
    d = to_dev(inp, cuda_device)
    for parts in (0, 1, 7):
        assert_close(run(d, inp, num_partitions=parts), ref, f"G={G} {dtype} parts={parts}")


@pytest.mark.parametrize("bs", [16, 32, 64])
def test_block_sizes_ragged_and_empty(cuda_device, bs):
    inp = workloads.make(kv8(5, 8, 2, bs, (15, 16, 0, 17, 513), seed=bs))
    ref = ref_of(inp)
    d = to_dev(inp, cuda_device)
    for parts in (0, 3, 40):
        out = run(d, inp, num_partitions=parts)
        assert_close(out, ref, f"bs={bs} parts={parts}")
        assert torch.all(out[2] == 0)


def test_scales_other_than_powers_of_two(cuda_device):
    inp = workloads.make(kv8(4, 32, 8, 16, (100, 1000, 2049, 7), seed=9))
    ref = ref_of(inp, k_scale=0.0137, v_scale=0.211)
    d = to_dev(inp, cuda_device)
    assert_close(run(d, inp, k_scale=0.0137, v_scale=0.211), ref, "scales")


def test_scaled_down_fp8_workload(cuda_device):
    inp = workloads.make(workloads.get("gqa_fp8", batch=6))
    assert_close(run(to_dev(inp, cuda_device), inp), ref_of(inp), "gqa_fp8 B6")


def test_out_of_range_block_id_is_reported(cuda_device):
    inp = workloads.make(kv8(2, 8, 2, 16, (200, 130), seed=5))
    d = to_dev(inp, cuda_device)
    bt = d["block_table"].clone()
    bt[0, 1] = inp["num_blocks"] + 3
    pa().device_status(reset=True)
    pa().decode_kv8(d["q"], d["k_cache"], d["v_cache"], bt, d["context_lens"], inp["scale"],
                    inp["k_scale"], inp["v_scale"])
    assert pa().device_status(reset=True) == pa().PA_ERR_BAD_BLOCK_ID
    assert_close(run(d, inp), ref_of(inp), "after error")


@pytest.mark.slow
def test_full_size_fp8_sampled(cuda_device):
    w = workloads.get("gqa_fp8")
    inp = workloads.make(w)
    out = run(to_dev(inp, cuda_device), inp)
    g = torch.Generator().manual_seed(0)
    cl = inp["context_lens"]
    bs_ = [int(cl.argmax()), int(cl.argmin())] + torch.randint(0, w.batch, (46,), generator=g).tolist()
    hs = torch.randint(0, w.num_q_heads, (48,), generator=g).tolist()
    pairs = np.array(list(zip(bs_, hs)), np.int32)
    assert_close(out[pairs[:, 0], pairs[:, 1]], ref_of(inp, pairs=pairs), "gqa_fp8 full")


def test_subnormal_codes_are_exact(cuda_device):
    # every key / value code subnormal (exponent field 0): with scales 2^7 they
    # carry values up to 1.75, so any loss of the smallest codes would show
    inp = workloads.make(kv8(3, 8, 2, 16, (40, 333, 5), seed=11))
    g = torch.Generator().manual_seed(3)
    for name in ("k_cache", "v_cache"):
        c = torch.randint(0, 8, inp[name].shape, generator=g, dtype=torch.int32)
        sign = torch.randint(0, 2, inp[name].shape, generator=g, dtype=torch.int32) << 7
        inp[name] = (c | sign).to(torch.uint8)
    ref = ref_of(inp, k_scale=128.0, v_scale=128.0)
    d = to_dev(inp, cuda_device)
    for parts in (0, 5):
        assert_close(run(d, inp, k_scale=128.0, v_scale=128.0, num_partitions=parts), ref,
                     f"subnormal parts={parts}")


def test_partition_then_merge_equals_full_call(cuda_device):
    inp = workloads.make(kv8(5, 32, 8, 16, (100, 1000, 2049, 7, 333), seed=13))
    d = to_dev(inp, cuda_device)
    args = (d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["context_lens"], inp["scale"],
            inp["k_scale"], inp["v_scale"])
    full = pa().decode_kv8(*args, num_partitions=37)
    desc = pa().gqa_desc(d["q"], d["k_cache"], d["block_table"], 37)
    ws = torch.full((pa().workspace_size(desc),), 0xAB, dtype=torch.uint8, device=cuda_device)
    out = torch.empty_like(d["q"])
    for passes in ("partition", "merge"):
        pa().decode_kv8(*args, out=out, workspace=ws, num_partitions=37, passes=passes)
    torch.cuda.synchronize()
    assert pa().device_status() == 0
    assert torch.equal(out, full)
