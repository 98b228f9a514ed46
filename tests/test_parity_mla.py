"""GPU parity of the MLA (shared-latent) decode path against the float64 oracle.

128 heads read one 576-wide latent row per token; the value is its first 512
dims.  Same tolerance as the GQA tests: |gpu - oracle| <= 2e-3 + 1e-2 |oracle|.
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


def mla(ctx, seed=0, bs=64, pool="factor:1.3"):
    return workloads.MLAWorkload("t", len(ctx), 128, 576, 512, "bf16", bs,
                                 "fixed:" + ",".join(str(c) for c in ctx), pool, seed,
                                 scale=1.0 / 192 ** 0.5)


def ref_of(inp, pairs=None):
    return oracle.decode_mla(u16(inp["q"]), u16(inp["latent_cache"]), inp["block_table"].numpy(),
                             inp["context_lens"].numpy(), inp["scale"], inp["dtype"],
                             v_dim=inp["v_dim"], pairs=pairs)


def to_dev(inp, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def run(d, inp, **kw):
    out = pa().decode_mla(d["q"], d["latent_cache"], d["block_table"], d["context_lens"],
                          inp["scale"], v_dim=inp["v_dim"], **kw)
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


@pytest.fixture(scope="module")
def dev(cuda_device):
    return cuda_device


def test_small_contexts(dev):
    inp = workloads.make(mla((70, 129), seed=1))
    ref = ref_of(inp)
    d = to_dev(inp, dev)
    for parts in (1, 2, 0):
        assert_close(run(d, inp, num_partitions=parts), ref, f"parts={parts}")


def test_ragged_and_tiny_contexts(dev):
    inp = workloads.make(mla((1, 64, 65, 0, 127, 300), seed=2))
    ref = ref_of(inp)
    d = to_dev(inp, dev)
    for parts in (1, 3, 7, 0, 50):
        out = run(d, inp, num_partitions=parts)
        assert_close(out, ref, f"parts={parts}")
        assert torch.all(out[3] == 0)


@pytest.mark.parametrize("bs", [16, 32, 48, 64, 128])
def test_block_sizes(dev, bs):
    inp = workloads.make(mla((200, 1000, 63), seed=3, bs=bs))
    ref = ref_of(inp)
    d = to_dev(inp, dev)
    for parts in (0, 4):
        assert_close(run(d, inp, num_partitions=parts), ref, f"bs={bs} parts={parts}")


def test_piece_bounds_across_sequence_units(dev):
    # Every non-empty sequence opens the work stream with a few empty units (its
    # fixed cost) before its tiles, so piece bounds fall before, inside and after
    # those units, and some pieces hold only empty units.  Many short and long
    # sequences with explicit piece counts put bounds everywhere.
    g = np.random.default_rng(11)
    ctx = [int(x) for x in g.integers(1, 700, 18)] + [0, 96, 97, 191, 192]
    inp = workloads.make(mla(tuple(ctx), seed=5))
    ref = ref_of(inp)
    d = to_dev(inp, dev)
    for parts in (2, 9, 23, 40, 74, 150):
        assert_close(run(d, inp, num_partitions=parts), ref, f"parts={parts}")


def test_query_only_16_byte_aligned(dev):
    # Query rows are read 32 bytes at a time when the query is 32-byte aligned and
    # 16 bytes at a time otherwise; a query 16 bytes past an aligned base takes the
    # second path and must give the same bits.
    inp = workloads.make(mla((200, 1000, 63), seed=6))
    ref = ref_of(inp)
    d = to_dev(inp, dev)
    q = d["q"]
    big = torch.empty(q.numel() + 8, dtype=q.dtype, device=dev)
    q16 = big[8:].view(q.shape)
    q16.copy_(q)
    assert q16.data_ptr() % 32 == 16
    for parts in (0, 3):
        out = run(dict(d, q=q16), inp, num_partitions=parts)
        assert_close(out, ref, f"16-byte query parts={parts}")
        assert torch.equal(out, run(d, inp, num_partitions=parts))


def test_scaled_down_mla_workload(dev):
    inp = workloads.make(workloads.get("mla", batch=3))
    ref = ref_of(inp)
    assert_close(run(to_dev(inp, dev), inp), ref, "mla B3")


def test_partition_then_merge_equals_full_call(dev):
    inp = workloads.make(mla((300, 777, 64), seed=4))
    d = to_dev(inp, dev)
    full = run(d, inp, num_partitions=5)
    out = torch.empty_like(full)
    desc = pa().mla_desc(d["q"], d["latent_cache"], d["block_table"], 512, 5)
    ws = torch.empty(pa().workspace_size(desc), dtype=torch.uint8, device=dev)
    for passes in ("partition", "merge"):
        pa().decode_mla(d["q"], d["latent_cache"], d["block_table"], d["context_lens"],
                        inp["scale"], v_dim=512, out=out, workspace=ws, num_partitions=5,
                        passes=passes)
    torch.cuda.synchronize()
    assert torch.equal(out, full)


def test_repeat_calls_are_bitwise_deterministic(dev):
    inp = workloads.make(workloads.get("mla", batch=6))
    d = to_dev(inp, dev)
    assert torch.equal(run(d, inp), run(d, inp))


def test_out_of_range_block_id_is_reported(dev):
    inp = workloads.make(mla((200, 130), seed=5))
    d = to_dev(inp, dev)
    bt = d["block_table"].clone()
    bt[0, 1] = inp["num_blocks"] + 3
    pa().device_status(reset=True)
    pa().decode_mla(d["q"], d["latent_cache"], bt, d["context_lens"], inp["scale"], v_dim=512)
    assert pa().device_status(reset=True) == pa().PA_ERR_BAD_BLOCK_ID
    assert_close(run(d, inp), ref_of(inp), "after error")


@pytest.mark.slow
def test_full_size_mla_sampled(dev):
    w = workloads.get("mla")
    inp = workloads.make(w)
    out = run(to_dev(inp, dev), inp)
    g = torch.Generator().manual_seed(0)
    cl = inp["context_lens"]
    bs_ = [int(cl.argmax()), int(cl.argmin())] + torch.randint(0, w.batch, (30,), generator=g).tolist()
    hs = torch.randint(0, 128, (32,), generator=g).tolist()
    pairs = np.array(list(zip(bs_, hs)), np.int32)
    ref = ref_of(inp, pairs=pairs)
    assert_close(out[pairs[:, 0], pairs[:, 1]], ref, "mla full")


def test_batch_past_the_default_shared_memory_of_the_merge(dev):
    # 13000 one-tile sequences: the merge's tile-prefix table (B + 1 ints) is past
    # the 48 KB default, so the library raises the merge kernel's limit.  Inputs
    # are drawn on the device (seeded); the oracle gets the sampled sequences only.
    B, bs, H, Dk, Dv = 13000, 64, 128, 576, 512
    gd = torch.Generator(device=dev).manual_seed(21)
    q = torch.randn((B, H, Dk), generator=gd, device=dev).to(torch.bfloat16)
    lat = torch.randn((B, bs, Dk), generator=gd, device=dev).to(torch.bfloat16)
    g = torch.Generator().manual_seed(21)
    table = torch.randperm(B, generator=g).to(torch.int32).reshape(B, 1)
    cl = torch.randint(1, bs + 1, (B,), generator=g).to(torch.int32)
    scale = 1.0 / 192 ** 0.5
    out = pa().decode_mla(q, lat, table.to(dev), cl.to(dev), scale, v_dim=Dv)
    torch.cuda.synchronize()
    assert pa().device_status() == 0
    seqs = [0, B - 1] + torch.randint(0, B, (10,), generator=g).tolist()
    blocks = table[seqs, 0].long()
    q_s = q[seqs].cpu()
    lat_s = lat[blocks.to(dev)].cpu()
    table_s = torch.arange(len(seqs), dtype=torch.int32).reshape(-1, 1)
    heads = torch.randint(0, H, (len(seqs),), generator=g).tolist()
    pairs = np.array(list(zip(range(len(seqs)), heads)), np.int32)
    ref = oracle.decode_mla(u16(q_s), u16(lat_s), table_s.numpy(), cl[seqs].numpy(), scale,
                            "bf16", v_dim=Dv, pairs=pairs)
    got = out[torch.tensor(seqs), torch.tensor(heads)]
    assert_close(got, ref, "B=13000")
