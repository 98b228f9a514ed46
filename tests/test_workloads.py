"""Host-side checks of the seeded workload generator (no attention arithmetic)."""
import math

import torch

import workloads


def test_tiny_workload_matches_its_description():
    inp = workloads.make(workloads.get("tiny"))
    assert inp["context_lens"].tolist() == [17, 40]
    assert inp["num_blocks"] == 8
    t = inp["block_table"]
    used = t[t >= 0].tolist()
    assert len(used) == 2 + 3 and len(set(used)) == 5 and all(0 <= x < 8 for x in used)
    assert inp["q"].dtype == torch.float16 and inp["k_cache"].shape == (8, 4, 16, 64)
    assert abs(inp["scale"] - 1 / 8) < 1e-15


def test_generation_is_seeded():
    a = workloads.make(workloads.get("gqa", batch=3))
    b = workloads.make(workloads.get("gqa", batch=3))
    for k in ("q", "k_cache", "v_cache", "block_table", "context_lens"):
        assert torch.equal(a[k], b[k])


def test_block_tables_are_disjoint_and_cover_each_context():
    for name in ("gqa", "mixed"):
        w = workloads.get(name, batch=16)
        inp = workloads.make(w)
        t, cl = inp["block_table"], inp["context_lens"]
        ids = []
        for b in range(w.batch):
            n = (int(cl[b]) + w.block_size - 1) // w.block_size
            assert bool((t[b, :n] >= 0).all()) and bool((t[b, n:] == -1).all())
            ids += t[b, :n].tolist()
        assert len(ids) == len(set(ids))
        assert max(ids) < inp["num_blocks"]


def test_context_distributions_stay_in_range():
    g = torch.Generator().manual_seed(0)
    u = workloads.draw_context_lens("uniform:512,4096", 10000, g)
    assert int(u.min()) >= 512 and int(u.max()) <= 4096
    lg = workloads.draw_context_lens("loguniform:1,32768", 20000, g)
    assert int(lg.min()) >= 1 and int(lg.max()) <= 32768
    # log-uniform: the median sits near sqrt(32768) ~ 181
    med = float(lg.float().median())
    assert 120 < med < 260, med
    # mean of floor(exp(U(0, ln 32768))) ~ (32768 - 1) / ln 32768
    assert abs(float(lg.float().mean()) - 32767 / math.log(32768)) < 200


def test_kv_bytes_accounting():
    w = workloads.get("gqa")
    cl = torch.tensor([10, 20], dtype=torch.int32)
    assert workloads.kv_bytes(w, cl) == 30 * 8 * 128 * 2 * 2
    m = workloads.get("mla")
    assert workloads.kv_bytes(m, cl) == 30 * 576 * 2


def test_index_list_workload_structure():
    # a scaled-down copy of the topk recipe: sorted unique draws below ctx - window,
    # then the window; only blocks holding a selected token are mapped, each once
    w = workloads.IndexedWorkload("t", 3, 8, 2, 128, "bf16", 16, 700, 60, 16, 5)
    inp = workloads.make_indexed(w)
    sel, table, bs = inp["token_index"], inp["block_table"], w.block_size
    assert sel.shape == (3, 76) and torch.all(inp["n_sel"] == 76)
    seen = set()
    for b in range(3):
        top, win = sel[b, :60], sel[b, 60:]
        assert torch.all(top[1:] > top[:-1]) and int(top.min()) >= 0 and int(top.max()) < 700 - 16
        assert win.tolist() == list(range(700 - 16, 700))
        need = set((sel[b] // bs).tolist())
        mapped = {j for j in range(table.shape[1]) if int(table[b, j]) >= 0}
        assert mapped == need
        ids = [int(table[b, j]) for j in mapped]
        assert not (set(ids) & seen) and len(set(ids)) == len(ids)
        seen |= set(ids)
    assert seen == set(range(inp["k_cache"].shape[0]))


def test_float8_workload_codes_are_finite_e4m3():
    w = workloads.get("gqa_fp8", batch=2)
    inp = workloads.make(w)
    for name in ("k_cache", "v_cache"):
        codes = inp[name]
        assert codes.dtype == torch.uint8
        assert not torch.any((codes & 0x7F) == 0x7F)          # no NaN code
        vals = codes.view(torch.float8_e4m3fn).float() * inp["k_scale"]
        assert abs(vals.mean().item()) < 0.05 and 0.8 < vals.std().item() < 1.2
