"""CPU checks of bench.py's output contract on its reference arm (the float64
oracle timed on host cores): one JSON line with the required keys, alone and
under torchrun with two ranks, where rank 0 alone prints."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REQUIRED = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
            "cpu_baseline", "e2e")


def json_lines(out):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def check_line(j, n_gpus):
    for k in REQUIRED:
        assert k in j, k
    assert j["impl"] == "reference" and j["n_gpus"] == n_gpus and j["steps"] == 2
    assert j["value"] > 0 and j["higher_is_better"] is True and j["dtype"] == "f64"
    assert "workload" in j["config"]
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == j["value"]
    e = j["e2e"]
    assert e["value"] == j["value"] and e["unit"] == j["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2",
                        "--warmup", "3", "--workload", "tiny"], cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1
    check_line(lines[0], 1)


def test_reference_arm_under_two_ranks():
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
                        "--master-port", "29541", "bench.py", "--impl", "reference", "--gpus", "2",
                        "--steps", "2", "--warmup", "3", "--workload", "tiny"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1                   # rank 0 alone prints
    check_line(lines[0], 2)


def test_cpu_baseline_reports_all_cores_and_one_thread():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    import workloads
    w = workloads.get("tiny")
    cb = bench.cpu_baseline(w, workloads.make(w), 0.2)
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0
    assert cb["value_1thread"] > 0 and "1 thread" in cb["sample_1thread"]


def test_parity_sample_against_the_oracle():
    import importlib.util
    import numpy as np
    import torch
    spec = importlib.util.spec_from_file_location("bench_mod2", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    import oracle
    import workloads
    w = workloads.get("gqa", batch=3)
    inp = workloads.make(w)
    u16 = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    full = oracle.decode(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]),
                         inp["block_table"].numpy(), inp["context_lens"].numpy(), inp["scale"],
                         inp["dtype"])
    exact = torch.from_numpy(np.asarray(full)).to(torch.bfloat16)   # the oracle, rounded
    r = bench.parity_sample(w, inp, exact.float(), n=12)
    assert r["within_tolerance"] and r["max_abs"] <= 2e-2 and r["rows"] == 12
    bad = exact.float().clone()
    bad[:, :, 5] += 0.5                                              # a wrong dim everywhere
    r = bench.parity_sample(w, inp, bad, n=12)
    assert not r["within_tolerance"] and r["max_abs"] >= 0.49
