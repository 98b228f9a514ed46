"""GPU parity of the GQA/MHA/MQA decode path against the float64 oracle.

Every case draws seeded inputs on the CPU, runs the CUDA library through its C
ABI (via the thin binding) and compares element by element with the oracle:
|gpu - oracle| <= 2e-3 + 1e-2 |oracle| (fp16/bf16 I/O, fp32 accumulation; the
page gather itself is index-exact).  Full-size workloads are checked on sampled
(sequence, head) rows that the oracle computes one by one, in the launch
configuration the bench times (default partition count).
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


def oracle_ref(inp, pairs=None):
    return oracle.decode(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]),
                         inp["block_table"].numpy(), inp["context_lens"].numpy(), inp["scale"],
                         inp["dtype"], pairs=pairs)


def run_gpu(d, scale, **kw):
    out = pa().decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["context_lens"],
                      scale, **kw)
    torch.cuda.synchronize()
    assert pa().device_status() == 0
    return out


def assert_close(gpu, ref, what=""):
    g = gpu.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), (f"{what}: {int(bad.sum())}/{bad.size} outside tolerance, "
                           f"max abs {err.max():.3e}")
    assert np.isfinite(g).all()


def gqa(B, Hq, Hkv, D, bs, ctx, dtype="bf16", seed=0, pool="factor:1.5"):
    return workloads.GQAWorkload("t", B, Hq, Hkv, D, dtype, bs,
                                 "fixed:" + ",".join(str(c) for c in ctx), pool, seed)


@pytest.fixture(scope="module")
def dev(cuda_device):
    return cuda_device


def test_tiny_workload(dev):
    inp = workloads.make(workloads.get("tiny"))
    ref = oracle_ref(inp)
    d = to_dev(inp, dev)
    for parts in (0, 1, 2, 3, 5, 64, 1000):
        assert_close(run_gpu(d, inp["scale"], num_partitions=parts), ref, f"parts={parts}")


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("D", [64, 128])
def test_group_sizes_and_head_dims(dev, G, D):
    Hkv = 2
    w = gqa(3, G * Hkv, Hkv, D, 16, (1, 77, 300), seed=G * 10 + D)
    inp = workloads.make(w)
    ref = oracle_ref(inp)
    d = to_dev(inp, dev)
    for parts in (0, 1, 7):
        assert_close(run_gpu(d, inp["scale"], num_partitions=parts), ref, f"G={G} D={D} p={parts}")


@pytest.mark.parametrize("bs", [16, 32, 64, 128])
def test_block_sizes(dev, bs):
    w = gqa(4, 8, 2, 128, bs, (15, 16, 17, 513), seed=bs)
    inp = workloads.make(w)
    ref = oracle_ref(inp)
    d = to_dev(inp, dev)
    for parts in (0, 3, 40):
        assert_close(run_gpu(d, inp["scale"], num_partitions=parts), ref, f"bs={bs} p={parts}")


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_dtypes(dev, dtype):
    w = gqa(3, 32, 8, 128, 16, (100, 1000, 2049), dtype=dtype, seed=5)
    inp = workloads.make(w)
    ref = oracle_ref(inp)
    out = run_gpu(to_dev(inp, dev), inp["scale"])
    assert out.dtype == (torch.float16 if dtype == "f16" else torch.bfloat16)
    assert_close(out, ref, dtype)


def test_empty_and_ragged_sequences(dev):
    w = gqa(6, 16, 4, 128, 16, (0, 1, 16, 0, 33, 250), seed=6)
    inp = workloads.make(w)
    ref = oracle_ref(inp)
    d = to_dev(inp, dev)
    for parts in (0, 1, 2, 9, 500):
        out = run_gpu(d, inp["scale"], num_partitions=parts)
        assert_close(out, ref, f"parts={parts}")
        assert torch.all(out[0] == 0) and torch.all(out[3] == 0)


def test_all_sequences_empty(dev):
    w = gqa(3, 8, 2, 64, 16, (0, 0, 0), seed=7)
    inp = workloads.make(w)
    d = to_dev(inp, dev)
    out = torch.full_like(d["q"], 7.0)
    out = pa().decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["context_lens"],
                      inp["scale"], out=out)
    torch.cuda.synchronize()
    assert torch.all(out == 0)


def test_scaled_down_gqa_workload(dev):
    inp = workloads.make(workloads.get("gqa", batch=6))
    ref = oracle_ref(inp)
    d = to_dev(inp, dev)
    for parts in (0, 13, 148):
        assert_close(run_gpu(d, inp["scale"], num_partitions=parts), ref, f"parts={parts}")


def test_scaled_down_mixed_workload(dev):
    inp = workloads.make(workloads.get("mixed", batch=24))
    ref = oracle_ref(inp)
    assert_close(run_gpu(to_dev(inp, dev), inp["scale"]), ref, "mixed")


def test_long_context_one_sequence(dev):
    inp = workloads.make(workloads.get("long", batch=1))
    ref = oracle_ref(inp)
    assert_close(run_gpu(to_dev(inp, dev), inp["scale"]), ref, "long")


def test_partition_then_merge_equals_full_call(dev):
    inp = workloads.make(workloads.get("gqa", batch=5))
    d = to_dev(inp, dev)
    full = run_gpu(d, inp["scale"], num_partitions=37)
    desc = pa().gqa_desc(d["q"], d["k_cache"], d["block_table"], 37)
    ws = torch.full((pa().workspace_size(desc),), 0xAB, dtype=torch.uint8, device=dev)  # garbage
    out = torch.empty_like(d["q"])
    for _ in range(2):
        for passes in ("partition", "merge"):
            pa().decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["context_lens"],
                        inp["scale"], out=out, workspace=ws, num_partitions=37, passes=passes)
        torch.cuda.synchronize()
        assert torch.equal(out, full)


def test_repeat_calls_are_bitwise_deterministic(dev):
    inp = workloads.make(workloads.get("mixed", batch=12))
    d = to_dev(inp, dev)
    a = run_gpu(d, inp["scale"])
    b = run_gpu(d, inp["scale"])
    assert torch.equal(a, b)


def test_permuted_pool_gives_identical_output(dev):
    inp = workloads.make(workloads.get("gqa", batch=4))
    d = to_dev(inp, dev)
    a = run_gpu(d, inp["scale"], num_partitions=1)
    nb = inp["k_cache"].shape[0]
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(3))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(nb)
    t2 = inp["block_table"].clone()
    m = t2 >= 0
    t2[m] = inv[t2[m].long()].to(torch.int32)
    b = pa().decode(d["q"], inp["k_cache"][perm].contiguous().to(dev),
                    inp["v_cache"][perm].contiguous().to(dev), t2.to(dev), d["context_lens"],
                    inp["scale"], num_partitions=1)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_out_of_range_block_id_is_reported_not_read(dev):
    w = gqa(2, 8, 2, 128, 16, (40, 40), seed=9)
    inp = workloads.make(w)
    d = to_dev(inp, dev)
    bt = d["block_table"].clone()
    bt[1, 1] = inp["num_blocks"] + 5           # outside the pool: must not be dereferenced
    pa().device_status(reset=True)
    pa().decode(d["q"], d["k_cache"], d["v_cache"], bt, d["context_lens"], inp["scale"])
    assert pa().device_status(reset=True) == pa().PA_ERR_BAD_BLOCK_ID
    # the device stays usable and a valid call succeeds afterwards
    ref = oracle_ref(inp)
    assert_close(run_gpu(d, inp["scale"]), ref, "after error")


def test_context_longer_than_table_is_reported(dev):
    w = gqa(2, 8, 2, 128, 16, (40, 40), seed=10)
    inp = workloads.make(w)
    d = to_dev(inp, dev)
    cl = d["context_lens"].clone()
    cl[0] = inp["max_blocks_per_seq"] * 16 + 1
    pa().device_status(reset=True)
    pa().decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], cl, inp["scale"])
    assert pa().device_status(reset=True) == pa().PA_ERR_BAD_BLOCK_ID


def _sampled_full_size(name, dev, n_pairs=48, seed=0):
    w = workloads.get(name)
    inp = workloads.make(w)
    d = to_dev(inp, dev)
    out = run_gpu(d, inp["scale"])            # default partitions = the bench's launch
    g = torch.Generator().manual_seed(seed)
    B, Hq = w.batch, w.num_q_heads
    # always include the longest and the shortest sequence, plus random rows
    cl = inp["context_lens"]
    bs = [int(cl.argmax()), int(cl.argmin())] + torch.randint(0, B, (n_pairs - 2,), generator=g).tolist()
    hs = torch.randint(0, Hq, (n_pairs,), generator=g).tolist()
    pairs = np.array(list(zip(bs, hs)), np.int32)
    ref = oracle_ref(inp, pairs=pairs)
    got = out[pairs[:, 0], pairs[:, 1]]
    assert_close(got, ref, name)


@pytest.mark.slow
def test_full_size_gqa_sampled(dev):
    _sampled_full_size("gqa", dev)


@pytest.mark.slow
def test_full_size_long_sampled(dev):
    _sampled_full_size("long", dev, n_pairs=16)


@pytest.mark.slow
def test_full_size_mixed_sampled(dev):
    _sampled_full_size("mixed", dev)


def test_maximum_batch(dev):
    # 4096 sequences (the largest batch): the tile prefix of every kernel fills
    # its shared-memory table; lengths 0..40 leave many segments unsplit and
    # some empty
    g = torch.Generator().manual_seed(11)
    ctx = torch.randint(0, 41, (4096,), generator=g).tolist()
    w = gqa(4096, 8, 2, 64, 16, ctx, seed=11)
    inp = workloads.make(w)
    d = to_dev(inp, dev)
    out = run_gpu(d, inp["scale"])
    rows = torch.randint(0, 4096, (40,), generator=g).tolist() + [4095, 0]
    heads = torch.randint(0, 8, (42,), generator=g).tolist()
    pairs = np.array(list(zip(rows, heads)), np.int32)
    assert_close(out[pairs[:, 0], pairs[:, 1]], oracle_ref(inp, pairs=pairs), "B=4096")
    for b in range(4096):
        if ctx[b] == 0:
            assert torch.all(out[b] == 0)
            break
