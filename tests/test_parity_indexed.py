"""GPU parity of the index-list decode against the float64 oracle.

Each sequence attends over a given list of its token positions (sorted uniform
draws plus a trailing window, or arbitrary orders and repeats); the kernel
gathers the selected rows itself.  Same tolerance as the other parity tests.
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


def small(B=3, Hq=8, Hkv=2, ctx=700, top=60, window=16, seed=0, dtype="bf16", bs=16):
    return workloads.IndexedWorkload("t", B, Hq, Hkv, 128, dtype, bs, ctx, top, window, seed)


def ref_of(inp, pairs=None, token_index=None, n_sel=None):
    ti = inp["token_index"] if token_index is None else token_index
    ns = inp["n_sel"] if n_sel is None else n_sel
    return oracle.decode_indexed(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]),
                                 inp["block_table"].numpy(), ti.numpy(), ns.numpy(),
                                 inp["scale"], inp["dtype"], pairs=pairs)


def run(d, inp, token_index=None, n_sel=None, **kw):
    out = pa().decode_indexed(d["q"], d["k_cache"], d["v_cache"], d["block_table"],
                              d["token_index"] if token_index is None else token_index,
                              d["n_sel"] if n_sel is None else n_sel, inp["scale"], **kw)
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


@pytest.mark.parametrize("G", [1, 4, 16])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_group_sizes_and_dtypes(cuda_device, G, dtype):
    inp = workloads.make_indexed(small(Hq=2 * G, seed=G, dtype=dtype))
    ref = ref_of(inp)
    d = to_dev(inp, cuda_device)
    for parts in (0, 1, 7, 40):
        assert_close(run(d, inp, num_partitions=parts), ref, f"G={G} {dtype} parts={parts}")


@pytest.mark.parametrize("bs", [16, 32, 64])
def test_block_sizes_and_ragged_counts(cuda_device, bs):
    inp = workloads.make_indexed(small(bs=bs, seed=bs))
    ns = torch.tensor([1, 0, 37], dtype=torch.int32)
    ref = ref_of(inp, n_sel=ns)
    d = to_dev(inp, cuda_device)
    for parts in (0, 3):
        out = run(d, inp, n_sel=ns.to(cuda_device), num_partitions=parts)
        assert_close(out, ref, f"bs={bs} parts={parts}")
        assert torch.all(out[1] == 0)


def test_unsorted_list_with_repeats(cuda_device):
    inp = workloads.make_indexed(small(seed=4))
    g = torch.Generator().manual_seed(9)
    ti = inp["token_index"].clone()
    for b in range(ti.shape[0]):
        ti[b] = ti[b][torch.randperm(ti.shape[1], generator=g)]
        ti[b, 5] = ti[b, 3]                                   # one position listed twice
    ref = ref_of(inp, token_index=ti)
    d = to_dev(inp, cuda_device)
    assert_close(run(d, inp, token_index=ti.to(cuda_device)), ref, "unsorted + repeat")


def test_bad_position_is_reported(cuda_device):
    inp = workloads.make_indexed(small(seed=5))
    d = to_dev(inp, cuda_device)
    ti = d["token_index"].clone()
    ti[0, 3] = inp["max_blocks_per_seq"] * 16 + 5             # past the table
    pa().device_status(reset=True)
    pa().decode_indexed(d["q"], d["k_cache"], d["v_cache"], d["block_table"], ti, d["n_sel"],
                        inp["scale"])
    assert pa().device_status(reset=True) == pa().PA_ERR_BAD_BLOCK_ID
    assert_close(run(d, inp), ref_of(inp), "after error")


@pytest.mark.slow
def test_full_size_topk_sampled(cuda_device):
    w = workloads.INDEXED["topk"]
    inp = workloads.make_indexed(w)
    out = run(to_dev(inp, cuda_device), inp)
    g = torch.Generator().manual_seed(0)
    bs_ = torch.randint(0, w.batch, (40,), generator=g).tolist()
    hs = torch.randint(0, w.num_q_heads, (40,), generator=g).tolist()
    pairs = np.array(list(zip(bs_, hs)), np.int32)
    assert_close(out[pairs[:, 0], pairs[:, 1]], ref_of(inp, pairs=pairs), "topk full")


def test_partition_then_merge_equals_full_call(cuda_device):
    inp = workloads.make_indexed(small(B=4, ctx=900, top=80, seed=14))
    d = to_dev(inp, cuda_device)
    args = (d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["token_index"], d["n_sel"],
            inp["scale"])
    full = pa().decode_indexed(*args, num_partitions=29)
    desc = pa().gqa_desc(d["q"], d["k_cache"], d["block_table"], 29)
    ws = torch.full((pa().workspace_size(desc),), 0xAB, dtype=torch.uint8, device=cuda_device)
    out = torch.empty_like(d["q"])
    for passes in ("partition", "merge"):
        pa().decode_indexed(*args, out=out, workspace=ws, num_partitions=29, passes=passes)
    torch.cuda.synchronize()
    assert pa().device_status() == 0
    assert torch.equal(out, full)
