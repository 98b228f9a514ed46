"""Pins for the float64 oracle: closed forms, invariants and brute force.

None of these re-types the oracle's formula: each checks the oracle against a
fact the definition of softmax attention or the Flash-Decoding split/merge
fixes independently (a special case with a closed form, an exact invariance, a
high-precision brute force written differently, a library decoder).
"""
import math
import os

import mpmath
import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def draw(B=3, Hq=4, Hkv=2, D=8, bs=4, ctx=(5, 9, 1), dtype="bf16", seed=0, pool_extra=3):
    w = workloads.GQAWorkload("t", B, Hq, Hkv, D, dtype, bs,
                              "fixed:" + ",".join(str(c) for c in ctx),
                              f"factor:{1 + pool_extra / 10}", seed)
    return workloads.make(w)


def run(inp, **kw):
    return oracle.decode(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]),
                         inp["block_table"].numpy(), inp["context_lens"].numpy(),
                         inp["scale"], inp["dtype"], **kw)


# ---------------------------------------------------------------- 16-bit decoding

def test_f16_decoding_matches_numpy_for_every_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_decoding_matches_torch_for_every_pattern():
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_f64(int(b) & 0xFFFF) for b in bits.tolist()])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ---------------------------------------------------------------- closed forms

def _golden():
    spec = {}
    with open(os.path.join(GOLDEN, "worked_example.txt")) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            k, v = line.split(":", 1)
            spec[k.strip()] = v.strip()
    return spec


def test_worked_example_closed_form():
    g = _golden()
    n, bs = int(g["context_len"]), int(g["block_size"])
    table = [int(x) for x in g["block_table"].split()]
    q = [float(x) for x in g["q"].split()]
    K = [[float(x) for x in r.split()] for r in g["K"].split("|")]
    V = [[float(x) for x in r.split()] for r in g["V"].split("|")]
    D = len(q)
    nb = len(table)
    kc = np.zeros((nb, 1, bs, D), np.float16)
    vc = np.zeros((nb, 1, bs, D), np.float16)
    for t in range(n):
        kc[table[t // bs], 0, t % bs] = K[t]
        vc[table[t // bs], 0, t % bs] = V[t]
    out = oracle.decode(np.array([[q]], np.float16), kc, vc, np.array([table], np.int32),
                        np.array([n], np.int32), 1.0, "f16")
    e = math.e
    want = [eval(x, {"e": e}) for x in g["expected"].replace("^", "**").split("|")]
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-15, atol=0)
    split = oracle.decode_split(np.array([[q]], np.float16), kc, vc, np.array([table], np.int32),
                                np.array([n], np.int32), 1.0, "f16", split_len=2)
    np.testing.assert_allclose(split[0, 0], want, rtol=1e-15, atol=0)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_context_one_returns_v0_exactly(dtype):
    inp = draw(ctx=(1, 1, 1), dtype=dtype, seed=3)
    out = run(inp)
    for b in range(3):
        blk = int(inp["block_table"][b, 0])
        for h in range(4):
            v0 = inp["v_cache"][blk, h // 2, 0].to(torch.float64).numpy()
            assert np.array_equal(out[b, h], v0)


def test_zero_query_gives_mean_of_values():
    inp = draw(ctx=(7, 13, 2), seed=4)
    inp["q"].zero_()
    out = run(inp)
    for b, n in enumerate(inp["context_lens"].tolist()):
        for h in range(4):
            rows = [inp["v_cache"][int(inp["block_table"][b, t // 4]), h // 2, t % 4]
                    .to(torch.float64).numpy() for t in range(n)]
            mean = [math.fsum(r[d] for r in rows) / n for d in range(8)]
            np.testing.assert_allclose(out[b, h], mean, rtol=1e-14, atol=1e-15)


def test_identical_keys_give_mean_of_values():
    inp = draw(ctx=(6, 11, 3), seed=5)
    inp["k_cache"][:] = inp["k_cache"][0, 0, 0]  # every key row the same vector
    out = run(inp)
    for b, n in enumerate(inp["context_lens"].tolist()):
        for h in range(4):
            rows = [inp["v_cache"][int(inp["block_table"][b, t // 4]), h // 2, t % 4]
                    .to(torch.float64).numpy() for t in range(n)]
            mean = [math.fsum(r[d] for r in rows) / n for d in range(8)]
            np.testing.assert_allclose(out[b, h], mean, rtol=1e-14, atol=1e-15)


def test_zero_context_gives_zero_row():
    inp = draw(ctx=(0, 5, 0), seed=6)
    out = run(inp)
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert np.any(out[1] != 0)


# ---------------------------------------------------------------- brute force

def _brute(q, K, V, scale):
    """softmax(q K^T scale) V at 50 digits, no max subtraction, contiguous rows."""
    mpmath.mp.dps = 50
    s = [mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(float(a)) * mpmath.mpf(float(b))
                                         for a, b in zip(q, k)) for k in K]
    w = [mpmath.exp(x) for x in s]
    Z = mpmath.fsum(w)
    return [float(mpmath.fsum(wt * mpmath.mpf(float(v[d])) for wt, v in zip(w, V)) / Z)
            for d in range(len(V[0]))]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_on_contiguous_rows(seed):
    """Build contiguous K/V per sequence, scatter them into a permuted pool, and
    compare the oracle with a 50-digit brute force on the contiguous rows."""
    g = torch.Generator().manual_seed(100 + seed)
    B, Hq, Hkv, D, bs = 2, 4, 2, 8, 4
    ctx = [13, 6]
    nblk = [(c + bs - 1) // bs for c in ctx]
    nb = sum(nblk) + 2
    perm = torch.randperm(nb, generator=g).tolist()
    Kc = [torch.randn(c, Hkv, D, generator=g).to(torch.bfloat16) for c in ctx]
    Vc = [torch.randn(c, Hkv, D, generator=g).to(torch.bfloat16) for c in ctx]
    q = (2.0 * torch.randn(B, Hq, D, generator=g)).to(torch.bfloat16)
    kc = torch.randn(nb, Hkv, bs, D, generator=g).to(torch.bfloat16)  # junk in unused rows
    vc = torch.randn(nb, Hkv, bs, D, generator=g).to(torch.bfloat16)
    table = torch.full((B, max(nblk)), -1, dtype=torch.int32)
    pos = 0
    for b in range(B):
        for j in range(nblk[b]):
            table[b, j] = perm[pos]
            pos += 1
        for t in range(ctx[b]):
            kc[table[b, t // bs], :, t % bs] = Kc[b][t]
            vc[table[b, t // bs], :, t % bs] = Vc[b][t]
    scale = 0.37
    out = oracle.decode(u16(q), u16(kc), u16(vc), table.numpy(), np.array(ctx, np.int32),
                        scale, "bf16")
    for b in range(B):
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            want = _brute(q[b, h].float().tolist(), Kc[b][:, kv].float().tolist(),
                          Vc[b][:, kv].float().tolist(), scale)
            np.testing.assert_allclose(out[b, h], want, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("split_len", [1, 4, 8, 12, 7, 13, 64])
def test_split_then_merge_equals_unsplit(split_len):
    inp = draw(B=4, ctx=(13, 1, 29, 8), seed=7)
    full = run(inp)
    split = oracle.decode_split(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]),
                                inp["block_table"].numpy(), inp["context_lens"].numpy(),
                                inp["scale"], "bf16", split_len=split_len)
    np.testing.assert_allclose(split, full, rtol=1e-12, atol=1e-14)


def test_permuted_pool_is_bitwise_invariant():
    inp = draw(B=3, ctx=(17, 9, 30), bs=4, seed=8)
    out = run(inp)
    nb = inp["k_cache"].shape[0]
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(9))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(nb)
    k2 = inp["k_cache"][perm].contiguous()      # new block i holds old block perm[i]
    v2 = inp["v_cache"][perm].contiguous()
    t2 = inp["block_table"].clone()
    m = t2 >= 0
    t2[m] = inv[t2[m].long()].to(torch.int32)
    out2 = oracle.decode(u16(inp["q"]), u16(k2), u16(v2), t2.numpy(),
                         inp["context_lens"].numpy(), inp["scale"], "bf16")
    assert np.array_equal(out, out2)


def test_unused_table_entries_are_never_read():
    inp = draw(B=2, ctx=(5, 9), bs=4, seed=10)
    out = run(inp)
    t = inp["block_table"].clone()
    t[t < 0] = 10 ** 6   # would be out of range if read
    out2 = oracle.decode(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]), t.numpy(),
                         inp["context_lens"].numpy(), inp["scale"], "bf16")
    assert np.array_equal(out, out2)


def test_out_of_range_block_id_is_reported():
    inp = draw(B=2, ctx=(5, 9), bs=4, seed=11)
    t = inp["block_table"].clone()
    t[1, 1] = inp["k_cache"].shape[0]
    with pytest.raises(RuntimeError):
        oracle.decode(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]), t.numpy(),
                      inp["context_lens"].numpy(), inp["scale"], "bf16")


def test_gqa_equals_mha_with_duplicated_kv_heads():
    inp = draw(B=2, Hq=6, Hkv=2, ctx=(9, 14), bs=4, seed=12)
    out = run(inp)
    G = 3
    k2 = inp["k_cache"].repeat_interleave(G, dim=1).contiguous()
    v2 = inp["v_cache"].repeat_interleave(G, dim=1).contiguous()
    out2 = oracle.decode(u16(inp["q"]), u16(k2), u16(v2), inp["block_table"].numpy(),
                         inp["context_lens"].numpy(), inp["scale"], "bf16")
    assert np.array_equal(out, out2)


def test_scale_and_query_rescaling_cancel():
    inp = draw(ctx=(11, 4, 20), seed=13)
    out = run(inp)
    q2 = (inp["q"].float() * 4.0).to(torch.bfloat16)   # exact: power of two
    assert torch.equal(q2.float(), inp["q"].float() * 4.0)
    out2 = oracle.decode(u16(q2), u16(inp["k_cache"]), u16(inp["v_cache"]),
                         inp["block_table"].numpy(), inp["context_lens"].numpy(),
                         inp["scale"] / 4.0, "bf16")
    assert np.array_equal(out, out2)


def test_pairs_select_rows_bitwise():
    inp = draw(ctx=(11, 4, 20), seed=14)
    out = run(inp)
    pairs = np.array([[2, 3], [0, 0], [1, 2]], np.int32)
    sub = run(inp, pairs=pairs)
    for i, (b, h) in enumerate(pairs):
        assert np.array_equal(sub[i], out[b, h])


def test_mla_equals_single_kv_head_gqa_on_the_latent():
    w = workloads.MLAWorkload("t", 3, 4, 24, 16, "bf16", 4, "fixed:9,1,14", "factor:1.3", 15,
                              scale=0.2)
    inp = workloads.make(w)
    lat = inp["latent_cache"]
    out = oracle.decode_mla(u16(inp["q"]), u16(lat), inp["block_table"].numpy(),
                            inp["context_lens"].numpy(), 0.2, "bf16", v_dim=16)
    kv = lat.unsqueeze(1).contiguous()  # [NB, 1, bs, 24]: one kv head, K = V = latent
    ref = oracle.decode(u16(inp["q"]), u16(kv), u16(kv), inp["block_table"].numpy(),
                        inp["context_lens"].numpy(), 0.2, "bf16")
    assert np.array_equal(out, ref[:, :, :16])


# ---------------------------------------------------------------- float8 KV cache

def test_e4m3_decoding_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    mine = np.array([oracle.e4m3_to_f64(int(c)) for c in codes])
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert list(codes[nan]) == [0x7F, 0xFF]
    assert np.isnan(mine[nan]).all()
    assert np.array_equal(mine[~nan], ref[~nan])
    assert np.nanmax(mine) == 448.0 and oracle.e4m3_to_f64(1) == 2.0 ** -9


def _kv8_inputs(seed=0, ctx=(5, 9, 1, 17)):
    w = workloads.GQAWorkload("t", len(ctx), 4, 2, 16, "bf16", 4,
                              "fixed:" + ",".join(str(c) for c in ctx), "factor:1.3", seed,
                              kv_dtype="e4m3")
    return workloads.make(w)


def _run_kv8(inp, k_scale=None, v_scale=None, scale=None):
    return oracle.decode_kv8(u16(inp["q"]), inp["k_cache"].numpy(), inp["v_cache"].numpy(),
                             inp["k_scale"] if k_scale is None else k_scale,
                             inp["v_scale"] if v_scale is None else v_scale,
                             inp["block_table"].numpy(), inp["context_lens"].numpy(),
                             inp["scale"] if scale is None else scale, inp["dtype"])


def test_kv8_decode_equals_16bit_decode_of_the_dequantised_cache():
    # code x 2^-6 is exact in bfloat16 (3 fraction bits, exponent well in range),
    # so the float8 path must reproduce the pinned 16-bit definition bit for bit
    inp = _kv8_inputs()
    deq = lambda c: (c.view(torch.float8_e4m3fn).to(torch.float64) * inp["k_scale"])  # noqa: E731
    k16 = deq(inp["k_cache"]).to(torch.bfloat16)
    v16 = deq(inp["v_cache"]).to(torch.bfloat16)
    assert torch.equal(k16.to(torch.float64), deq(inp["k_cache"]))
    ref = oracle.decode(u16(inp["q"]), u16(k16), u16(v16), inp["block_table"].numpy(),
                        inp["context_lens"].numpy(), inp["scale"], inp["dtype"])
    assert np.array_equal(_run_kv8(inp), ref)


def test_kv8_key_scale_folds_into_the_softmax_scale():
    inp = _kv8_inputs(seed=1)
    a = _run_kv8(inp, k_scale=0.37, v_scale=1.0)
    b = _run_kv8(inp, k_scale=1.0, v_scale=1.0, scale=inp["scale"] * 0.37)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_kv8_value_scale_scales_the_output():
    inp = _kv8_inputs(seed=2)
    a = _run_kv8(inp, v_scale=0.37)
    b = _run_kv8(inp, v_scale=1.0) * 0.37
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- index-list decode

def _indexed_small(seed=0, ctx=200, top=20, window=8):
    w = workloads.IndexedWorkload("t", 3, 4, 2, 16, "bf16", 8, ctx, top, window, seed)
    return workloads.make_indexed(w)


def _run_indexed(inp, token_index=None, n_sel=None):
    return oracle.decode_indexed(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]),
                                 inp["block_table"].numpy(),
                                 (inp["token_index"] if token_index is None else token_index).numpy(),
                                 (inp["n_sel"] if n_sel is None else n_sel).numpy(),
                                 inp["scale"], inp["dtype"])


def test_indexed_decode_equals_dense_decode_of_the_gathered_rows():
    # brute force: copy the selected rows, in list order, into a fresh contiguous
    # paged cache and run the (pinned) dense definition over it
    inp = _indexed_small()
    B, bs = inp["q"].shape[0], 8
    k, v, bt, sel = inp["k_cache"], inp["v_cache"], inp["block_table"], inp["token_index"]
    n = sel.shape[1]
    nblk = (n + bs - 1) // bs
    kd = torch.zeros((B * nblk, k.shape[1], bs, k.shape[3]), dtype=k.dtype)
    vd = torch.zeros_like(kd)
    for b in range(B):
        for i, pos in enumerate(sel[b].tolist()):
            phys = int(bt[b, pos // bs])
            kd[b * nblk + i // bs, :, i % bs] = k[phys, :, pos % bs]
            vd[b * nblk + i // bs, :, i % bs] = v[phys, :, pos % bs]
    table = torch.arange(B * nblk, dtype=torch.int32).view(B, nblk)
    ref = oracle.decode(u16(inp["q"]), u16(kd), u16(vd), table.numpy(),
                        inp["n_sel"].numpy(), inp["scale"], inp["dtype"])
    assert np.array_equal(_run_indexed(inp), ref)


def test_indexed_decode_with_every_position_equals_dense_decode():
    inp = _indexed_small(seed=1, ctx=48, top=0, window=48)   # the whole context, in order
    ref = oracle.decode(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]),
                        inp["block_table"].numpy(), inp["context_lens"].numpy(), inp["scale"],
                        inp["dtype"])
    assert np.array_equal(_run_indexed(inp), ref)


def test_indexed_decode_ignores_the_order_of_the_list():
    inp = _indexed_small(seed=2)
    g = torch.Generator().manual_seed(5)
    shuffled = torch.stack([r[torch.randperm(r.numel(), generator=g)] for r in inp["token_index"]])
    np.testing.assert_allclose(_run_indexed(inp, token_index=shuffled), _run_indexed(inp),
                               rtol=1e-12, atol=1e-13)


def test_indexed_decode_reads_only_the_first_n_sel_entries():
    inp = _indexed_small(seed=3)
    ns = torch.tensor([5, 0, 28], dtype=torch.int32)
    poisoned = inp["token_index"].clone()
    poisoned[0, 5:] = -7
    poisoned[1, :] = 10 ** 6
    a = _run_indexed(inp, token_index=poisoned, n_sel=ns)
    b = _run_indexed(inp, n_sel=ns)
    assert np.array_equal(a, b)
    assert np.all(a[1] == 0)
