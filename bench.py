"""Benchmark of the paged split-KV decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload mixed|long|gqa|mla|tiny|gqa_fp8|topk] [--batch B]
                    [--impl ours|reference]

The default workload is the mixed continuous-batching decode (256 sequences,
lengths log-uniform in [1, 32768]), the largest single-GPU configuration; the
long-context one is `--workload long`.  --batch replaces the workload's batch
size (for profiling a smaller case of the same shapes and length mix).

One step = one paged decode call (partition pass + LSE merge pass) over the
workload's whole batch, inputs resident in HBM.  The L2 is flushed between
timed steps (a 512 MiB write, then a 512 MiB read of another buffer so that no
dirty lines are left to write back during the timed call); each step is timed
with CUDA events on the launching stream and the per-step times are summed.
Metric: effective KV-read GB/s = algorithmic KV bytes (every live K/V element
once) / step time; ms_per_step is the mean step time.

Multi-GPU (torchrun, one process per GPU): every rank decodes its own batch of
independent sequences (weak scaling, no collective on the data path); the step
time is the max over ranks and the value counts the bytes of all ranks.

--impl reference times the float64 CPU oracle (the only other implementation of
the operation) on a bounded sample of the same workload on this host's cores.
"""
from __future__ import annotations

import argparse
import re
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "paged decode attention: effective KV-read GB/s vs HBM peak; µs per decode step"
UNIT = "GB/s"
FLUSH_BYTES = 512 << 20

DESCRIPTIONS = {
    "tiny": "tiny paged decode: B2 Hq4 Hkv4 D64 fp16 bs16 ctx {17,40} 8-block pool",
    "gqa": "GQA decode: B32 Hq32 Hkv8 D128 bf16 bs16 ctx U[512,4096] pool 1.25x shuffled",
    "long": "long-context GQA decode: B4 Hq32 Hkv8 D128 bf16 bs64 ctx 131072 shuffled",
    "mla": "MLA absorbed decode: B64 H128 latent 576 (V = first 512) bf16 bs64 ctx U[1024,8192]",
    "mixed": "mixed continuous-batching decode: B256 Hq64 Hkv8 D128 bf16 bs16 ctx log-U[1,32768]",
    "gqa_fp8": "GQA decode over a float8 E4M3 KV cache (one scale per tensor): B32 Hq32 Hkv8 D128 "
               "bf16 q/out bs16 ctx U[512,4096] pool 1.25x shuffled",
    "topk": "index-list GQA decode: B32 Hq32 Hkv8 D128 bf16 bs16 ctx 32768, 1152 selected "
            "positions per sequence (1024 uniform + last 128), referenced blocks shuffled",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="mixed",
                    choices=sorted(list(workloads.WORKLOADS) + list(workloads.INDEXED)))
    ap.add_argument("--batch", type=int, default=None,
                    help="replace the workload's batch size (same shapes and length mix)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--sweep", choices=["mha", "mqa"], default=None,
                    help="sequence-length scaling sweep 512..64k (one JSON line per length)")
    ap.add_argument("--sweep-batch", type=int, default=1)
    ap.add_argument("--merge", choices=["separate", "fused"], default="separate",
                    help="16-bit GQA workloads: 'fused' times pa_decode_fused (the last piece "
                         "of each split segment merges it; one launch per step)")
    return ap.parse_args()


# ------------------------------------------------------------------ distributed

def dist_setup(n):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def get_workload(name, seed_offset=0, batch=None):
    import dataclasses
    w = workloads.INDEXED[name] if name in workloads.INDEXED else workloads.get(name)
    if batch is not None and batch != w.batch:
        if getattr(w, "ctx", "").startswith("fixed:"):
            raise SystemExit(f"--batch: workload {name} has fixed context lengths")
        w = dataclasses.replace(w, batch=batch)
    return dataclasses.replace(w, seed=w.seed + seed_offset) if seed_offset else w


def describe(name, batch=None):
    """The workload's description, with the batch size replaced when overridden."""
    d = DESCRIPTIONS[name]
    return re.sub(r"\bB\d+", f"B{batch}", d, count=1) if batch is not None else d


def workload_config(args, w, inp, world):
    """The `config` object of the JSON line: the workload and how it is timed.
    Both arms print the same keys and values for the same workload."""
    return {"workload": describe(args.workload, args.batch), "batch": w.batch,
            "kv_bytes_per_step_per_gpu": workloads.kv_bytes(w, live_lens(w, inp)),
            "tokens_per_step_per_gpu": int(live_lens(w, inp).sum()),
            "parallelism": f"replicas x{world} (independent batches)",
            "l2": "flushed between steps (512 MiB write + 512 MiB read of another buffer)"}


def make_inputs(w):
    return workloads.make_indexed(w) if w.kind == "gqa_indexed" else workloads.make(w)


def live_lens(w, inp):
    """Tokens each sequence attends over (the selected counts for an index list)."""
    return inp["n_sel"] if w.kind == "gqa_indexed" else inp["context_lens"]


def rank_workload(name, rank, world, batch=None):
    """The workload a rank decodes: the same shapes on every rank, its own seeded
    batch of independent sequences when several ranks run (weak scaling)."""
    return get_workload(name, 7919 * rank if world > 1 else 0, batch)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed loop runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.lines = []
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [l for (t, l) in self.lines if t0 - 0.06 <= t <= t1 + 0.06] or \
               [l for (_, l) in self.lines]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                smax.append(float(f[1]))
            except ValueError:
                continue
            for name, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ helpers

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs"), d.get("bf16_tflops"), d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def kernel_hash(files):
    """Hash of the kernel sources with comments and blank space removed: traffic
    counters stay valid across comment edits, and go stale on any code change."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "paged_split_kv_attention_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload, kernel_files):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel_hash") != kernel_hash(kernel_files):
        return None
    return e.get("dram_bytes_per_launch")


def oracle_rows(w, inp, pairs, nthreads):
    """The float64 oracle on the given (sequence, head) rows of this workload."""
    import numpy as np

    import oracle
    u16 = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    bt, cl = inp["block_table"].numpy(), inp["context_lens"].numpy()
    if w.kind == "gqa_indexed":
        return oracle.decode_indexed(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]), bt,
                                     inp["token_index"].numpy(), inp["n_sel"].numpy(),
                                     inp["scale"], inp["dtype"], pairs=pairs, nthreads=nthreads)
    if w.kind == "gqa" and getattr(w, "kv_dtype", None) == "e4m3":
        return oracle.decode_kv8(u16(inp["q"]), inp["k_cache"].numpy(), inp["v_cache"].numpy(),
                                 inp["k_scale"], inp["v_scale"], bt, cl, inp["scale"],
                                 inp["dtype"], pairs=pairs, nthreads=nthreads)
    if w.kind == "gqa":
        return oracle.decode(u16(inp["q"]), u16(inp["k_cache"]), u16(inp["v_cache"]), bt, cl,
                             inp["scale"], inp["dtype"], pairs=pairs, nthreads=nthreads)
    return oracle.decode_mla(u16(inp["q"]), u16(inp["latent_cache"]), bt, cl, inp["scale"],
                             inp["dtype"], w.v_dim, pairs=pairs, nthreads=nthreads)


def parity_sample(w, inp, out_host, n=32, seed=0):
    """Error of sampled output rows (the longest and shortest sequence plus random
    ones) against the float64 oracle, with the elementwise tolerance of the tests."""
    import numpy as np
    cl = live_lens(w, inp)
    H = w.num_heads if w.kind == "mla" else w.num_q_heads
    g = torch.Generator().manual_seed(seed)
    bs = [int(cl.argmax()), int(cl.argmin())] + torch.randint(0, w.batch, (n - 2,),
                                                              generator=g).tolist()
    hs = torch.randint(0, H, (n,), generator=g).tolist()
    pairs = np.array(list(zip(bs, hs)), np.int32)
    ref = np.asarray(oracle_rows(w, inp, pairs, os.cpu_count() or 1), np.float64)
    got = out_host[torch.from_numpy(pairs[:, 0]).long(),
                   torch.from_numpy(pairs[:, 1]).long()].double().numpy()
    err = np.abs(got - ref)
    big = np.abs(ref) >= 0.05
    return {"rows": n, "max_abs": float(err.max()),
            "max_rel": float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0,
            "within_tolerance": bool(np.all(err <= 2e-3 + 1e-2 * np.abs(ref))),
            "tolerance": "|out - oracle| <= 2e-3 + 1e-2 |oracle| elementwise (float64 oracle)"}


def size_sample(run, cl, batch, target_s):
    """Leading sequences of the batch that one oracle run covers in about target_s:
    the sample grows from the first sequence, each estimate of the time per token
    taken from the last run (a short first sequence alone overstates it), at least
    doubling each time.  Returns the sequence count and the last run's seconds."""
    nseq = 1
    dt = run(nseq)
    while nseq < batch and dt < 0.5 * target_s:
        per_tok = max(dt, 1e-4) / max(int(cl[:nseq].sum()), 1)
        k, acc = 0, 0.0
        while k < batch and acc + per_tok * int(cl[k]) <= target_s:
            acc += per_tok * int(cl[k])
            k += 1
        nseq = min(batch, max(k, 2 * nseq))
        dt = run(nseq)
    return nseq, dt


def cpu_baseline(w, inp, target_s):
    """Time the float64 oracle on a bounded sample (leading sequences of the batch)."""
    import numpy as np
    nthreads = os.cpu_count() or 1
    cl = live_lens(w, inp)
    H = w.num_heads if w.kind == "mla" else w.num_q_heads

    def run(nseq, nheads, threads=nthreads):
        pairs = np.array([(b, h) for b in range(nseq) for h in range(nheads)], np.int32)
        t0 = time.perf_counter()
        oracle_rows(w, inp, pairs, threads)
        return time.perf_counter() - t0

    # when the whole batch takes less than target_s, whole passes repeat until it is
    nseq, dt = size_sample(lambda k: run(k, H), cl, w.batch, target_s)
    reps = 1
    while nseq == w.batch and dt < target_s and reps < 1000:
        dt += run(nseq, H)
        reps += 1
    sample_cl = cl[:nseq]
    nbytes = workloads.kv_bytes(w, sample_cl) * reps
    # the same oracle on one thread, over the first sequence (all heads)
    t_one = max(run(1, H, threads=1), 1e-6)
    return {"value": nbytes / dt / 1e9, "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "sample": f"first {nseq} of {w.batch} sequences ({int(sample_cl.sum())} tokens, all "
                      f"{H} heads) x {reps} pass(es), float64 C oracle, {dt:.1f} s",
            "value_1thread": workloads.kv_bytes(w, cl[:1]) / t_one / 1e9,
            "sample_1thread": f"first sequence ({int(cl[0])} tokens, all {H} heads), 1 thread",
            "seconds": dt + t_one}


# ------------------------------------------------------------------ our implementation

def run_ours(args, rank, world, local):
    import paged_split_kv_attention_b200 as pa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = rank_workload(args.workload, rank, world, args.batch)
    inp = make_inputs(w)
    kv_bytes = workloads.kv_bytes(w, live_lens(w, inp))
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    scale = inp["scale"]
    stream = torch.cuda.current_stream(dev)

    kv8 = getattr(w, "kv_dtype", None) == "e4m3"
    if w.kind == "gqa_indexed":
        desc = pa.gqa_desc(d["q"], d["k_cache"], d["block_table"])
        out = torch.empty_like(d["q"])

        def call(passes):
            return pa.decode_indexed(d["q"], d["k_cache"], d["v_cache"], d["block_table"],
                                     d["token_index"], d["n_sel"], scale, out=out, workspace=ws,
                                     passes=passes)
        n_kernels = 1
        kernel_files = ["pa_gqa.cuh", "pa_device.cuh"]
        kname = "gqa_decode_kernel (index-list gathers)"
    elif w.kind == "gqa" and kv8:
        desc = pa.PADesc(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                         d["block_table"].shape[1], d["k_cache"].shape[0],
                         pa.PA_BF16 if w.dtype == "bf16" else pa.PA_F16, 0)
        out = torch.empty_like(d["q"])

        def call(passes):
            return pa.decode_kv8(d["q"], d["k_cache"], d["v_cache"], d["block_table"],
                                 d["context_lens"], scale, inp["k_scale"], inp["v_scale"],
                                 out=out, workspace=ws, passes=passes)
        n_kernels = 1
        kernel_files = ["pa_gqa.cuh", "pa_device.cuh"]
        kname = "gqa_decode_kernel (float8 KV)"
    elif w.kind == "gqa":
        desc = pa.gqa_desc(d["q"], d["k_cache"], d["block_table"])
        out = torch.empty_like(d["q"])
        call = lambda passes: pa.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"],  # noqa
                                        d["context_lens"], scale, out=out, workspace=ws,
                                        passes=passes)
        n_kernels = 1
        kernel_files = ["pa_gqa.cuh", "pa_device.cuh"]
        kname = "gqa_decode_kernel"
    else:
        desc = pa.mla_desc(d["q"], d["latent_cache"], d["block_table"], w.v_dim)
        out = torch.empty((w.batch, w.num_heads, w.v_dim), dtype=d["q"].dtype, device=dev)
        call = lambda passes: pa.decode_mla(d["q"], d["latent_cache"], d["block_table"],  # noqa
                                            d["context_lens"], scale, v_dim=w.v_dim, out=out,
                                            workspace=ws, passes=passes)
        n_kernels = 1
        kernel_files = ["pa_mla.cuh", "pa_tcgen05.cuh", "pa_device.cuh"]
        kname = "mla_decode_kernel"
    fused = args.merge == "fused"
    if fused and not (w.kind == "gqa" and not kv8):
        raise SystemExit("--merge fused applies to the 16-bit GQA workloads")
    step_passes = "fused" if fused else "both"
    if fused:
        kname = "gqa_decode_kernel (single-pass merge)"
    ws = torch.empty(pa.workspace_size(desc), dtype=torch.uint8, device=dev)
    parts = desc.num_partitions or pa.default_partitions(
        {"gqa": "gqa_fp8" if kv8 else "gqa", "gqa_indexed": "gqa_indexed"}.get(w.kind, "mla"),
        getattr(w, "head_dim", 128))
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=sink)

    for _ in range(args.warmup):
        flush()
        call(step_passes)
    torch.cuda.synchronize()
    if pa.device_status() != 0:
        raise RuntimeError("kernel reported an error during warm-up")

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(local) if torch.cuda.is_available() else None
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    # one step = pa_decode = the partition kernel + the merge kernel (the merge is
    # launched with programmatic dependent launch, so nothing may sit between them)
    for i in range(K):
        flush()
        ev[i][0].record(stream)
        call(step_passes)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(world)
    clocks = sampler.stop(t0, t1) if sampler else None
    step_ms = [a.elapsed_time(c) for a, _, c in ev]
    # the dominant kernel alone, for the roofline: same flush, events around the
    # partition kernel only (the merge runs after the second event; the
    # single-pass form has no merge launch, its one kernel is timed)
    Kp = min(K, 200)
    for i in range(Kp):
        flush()
        ev[i][0].record(stream)
        call("fused" if fused else "partition")
        ev[i][1].record(stream)
        if not fused:
            call("merge")
    torch.cuda.synchronize()
    part_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(Kp)]
    if pa.device_status() != 0:
        raise RuntimeError("kernel reported an error during the timed loop")
    local_total = sum(step_ms)
    total_ms = max_over_ranks(local_total, world, dev)
    all_bytes = sum_over_ranks(float(kv_bytes), world, dev)
    ms_per_step = total_ms / K
    value = all_bytes * K / (total_ms / 1e3) / 1e9

    # e2e: same call through the public API with host buffers, H2D + D2H inside the region
    e2e = None
    if not args.no_e2e:
        host = {k: v.pin_memory() for k, v in inp.items() if isinstance(v, torch.Tensor)}
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        dev_in = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = out_h.numel() * out_h.element_size()
        Ke = max(3, min(K, 20))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for it in range(2 + Ke):
            if it == 2:
                barrier(world)
                torch.cuda.synchronize()
                e0.record(stream)
            for k2, v in host.items():
                dev_in[k2].copy_(v, non_blocking=True)
            if w.kind == "gqa_indexed":
                pa.decode_indexed(dev_in["q"], dev_in["k_cache"], dev_in["v_cache"],
                                  dev_in["block_table"], dev_in["token_index"], dev_in["n_sel"],
                                  scale, out=out, workspace=ws)
            elif w.kind == "gqa" and kv8:
                pa.decode_kv8(dev_in["q"], dev_in["k_cache"], dev_in["v_cache"],
                              dev_in["block_table"], dev_in["context_lens"], scale,
                              inp["k_scale"], inp["v_scale"], out=out, workspace=ws)
            elif w.kind == "gqa":
                pa.decode(dev_in["q"], dev_in["k_cache"], dev_in["v_cache"], dev_in["block_table"],
                          dev_in["context_lens"], scale, out=out, workspace=ws,
                          passes=step_passes)
            else:
                pa.decode_mla(dev_in["q"], dev_in["latent_cache"], dev_in["block_table"],
                              dev_in["context_lens"], scale, v_dim=w.v_dim, out=out, workspace=ws)
            out_h.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": all_bytes * Ke / (e_ms / 1e3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "includes": "H2D of q, KV pool, block_table, context_lens from pinned host "
                           "memory + decode + D2H of out, per step"}

    hbm, tf, tf_sus, peak_src = measured_peaks()
    part_avg_s = statistics.mean(part_ms) / 1e3
    achieved = kv_bytes / part_avg_s / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4),
                "traffic": None if fused else profiled_traffic(args.workload, kernel_files),
                "kernel": kname, "kernel_us": round(part_avg_s * 1e6, 2),
                "peak_source": f"{peak_src} hbm_gbs (copy)",
                "nominal_frac_8tbs": round(achieved / 8000.0, 4)}
    if w.kind == "mla":
        # a dense contraction (~240 flop per latent byte): measured against the
        # tensor roofline; the step loop runs for seconds, so the sustained peak
        fl = workloads.flops(w, inp["context_lens"])
        tflops = fl / part_avg_s / 1e12
        roofline.update({"bound": "tensor", "achieved": round(tflops, 1), "peak": tf_sus,
                         "unit": "TFLOP/s", "frac": round(tflops / tf_sus, 4),
                         "flops_per_launch": int(fl),
                         "peak_source": f"{peak_src} bf16_tflops_sustained (cuBLAS)",
                         "hbm_gbs": round(achieved, 1), "hbm_frac": round(achieved / hbm, 4)})
        roofline.pop("nominal_frac_8tbs", None)

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "us_per_step": round(ms_per_step * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": inp["dtype"], "data": "synthetic (seeded N(0,1) q/K/V, shuffled block pool)",
        "config": workload_config(args, w, inp, world),
        "launch": {"partitions": parts,
                   "merge": ("single-pass (pa_decode_fused: one launch)" if fused else
                             "separate kernel (programmatic dependent launch)")},
        "roofline": roofline, "clocks": clocks, "e2e": e2e,
        "gpu_launches": (1 if fused else 2) * K,
        "gpu_launches_note": ("per step: the partition kernel, which also merges" if fused else
                              "per step: the partition kernel + the LSE merge kernel"),
    }
    if rank == 0 and world == 1:
        # the last step's output against the oracle on sampled rows (after all timing)
        try:
            result["parity"] = parity_sample(w, inp, out.float().cpu())
        except Exception as e:  # reported, never fatal to the measurement line
            result["parity"] = {"error": repr(e)[:200]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(w, inp, args.cpu_seconds)
        cb.pop("seconds", None)
        result["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------ reference arm

def run_reference(args, rank, world):
    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    import numpy as np

    w = get_workload(args.workload, batch=args.batch)
    inp = make_inputs(w)
    nthreads = os.cpu_count() or 1
    cl = live_lens(w, inp)
    H = w.num_heads if w.kind == "mla" else w.num_q_heads
    # each step: a bounded sample (leading sequences, all heads) sized to ~2 s of CPU work
    budget_per_step = max(0.5, min(3.0, 150.0 / max(1, args.steps + args.warmup)))

    def step(nseq):
        pairs = np.array([(b, h) for b in range(nseq) for h in range(H)], np.int32)
        t0 = time.perf_counter()
        oracle_rows(w, inp, pairs, nthreads)
        return time.perf_counter() - t0

    nseq, _ = size_sample(step, cl, w.batch, budget_per_step)
    for _ in range(args.warmup):
        step(nseq)
    times = [step(nseq) for _ in range(args.steps)]
    nbytes = workloads.kv_bytes(w, cl[:nseq])
    total = sum(times)
    value = nbytes * len(times) / total / 1e9
    sample = (f"first {nseq} of {w.batch} sequences ({int(cl[:nseq].sum())} tokens, all {H} "
              f"heads) per step, float64 C oracle")
    result = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / len(times) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) q/K/V, shuffled block pool)",
        "config": workload_config(args, w, inp, world),
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": nthreads,
                         "kind": "oracle", "sample": sample, "sample_sequences": nseq},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_sweep(args):
    """Sequence-length scaling, one JSON line per length: the split decode (default
    launch, the flattened tile stream cut over every warp of the GPU) beside the
    same kernel launched with one CTA per 8 (sequence, kv head) segments, i.e. no
    split across SMs (with 8 or more segments each warp takes one whole segment;
    with fewer, one CTA's warps share them as a one-block-per-head decode would),
    the baseline Flash-Decoding is measured against."""
    import paged_split_kv_attention_b200 as pa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    hbm, _, _, peak_src = measured_peaks()
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    K, W = max(3, min(args.steps, 100)), max(3, args.warmup)
    for ctx in workloads.SWEEP_CTX:
        w = workloads.scaling(args.sweep, ctx, args.sweep_batch)
        inp = workloads.make(w)
        kv_bytes = workloads.kv_bytes(w, inp["context_lens"])
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        out = torch.empty_like(d["q"])
        segments = w.batch * w.num_kv_heads
        res = {}
        for label, parts in (("split", 0), ("no_split", -(-segments // 8))):
            desc = pa.gqa_desc(d["q"], d["k_cache"], d["block_table"], parts)
            ws = torch.empty(pa.workspace_size(desc), dtype=torch.uint8, device=dev)
            times = []
            for it in range(W + K):
                flush_w.zero_()
                torch.sum(flush_r, dim=0, out=sink)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                pa.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["context_lens"],
                          inp["scale"], out=out, workspace=ws, num_partitions=parts)
                e1.record(stream)
                if it >= W:
                    times.append((e0, e1))
            torch.cuda.synchronize()
            if pa.device_status() != 0:
                raise RuntimeError("kernel reported an error")
            us = statistics.median(a.elapsed_time(b) for a, b in times) * 1e3
            res[label] = {"us_per_step": round(us, 2), "GB/s": round(kv_bytes / us / 1e3, 1),
                          "frac": round(kv_bytes / us / 1e3 / hbm, 4),
                          "partitions": parts or pa.default_partitions("gqa", 128)}
        print(json.dumps({
            "metric": METRIC, "sweep": args.sweep, "ctx": ctx, "batch": w.batch,
            "heads": {"q": w.num_q_heads, "kv": w.num_kv_heads, "dim": w.head_dim},
            "kv_bytes": kv_bytes, "split": res["split"], "no_split": res["no_split"],
            "speedup_split_vs_no_split": round(res["no_split"]["us_per_step"] /
                                               res["split"]["us_per_step"], 2),
            "peak": {"hbm_gbs": hbm, "source": peak_src}, "steps": K, "warmup": W,
            "l2": "flushed before every step", "data": "synthetic (seeded N(0,1))"}), flush=True)


def main():
    args = parse()
    if args.sweep:
        run_sweep(args)
        return
    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
