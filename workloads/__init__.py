"""Seeded synthetic workloads for paged decode attention.

This module only draws random inputs and builds block tables.  It holds none of
the attention arithmetic, so that both the float64 oracle and the GPU library
can consume its tensors without sharing any computation.

Every tensor is drawn on the CPU from a ``torch.Generator`` seeded per workload;
q/K/V values are float32 N(0, 1) draws rounded to the workload's 16-bit type, so
the oracle and the GPU see identical bits.  Physical blocks are handed out from
a seeded random permutation of the pool, in sequence order; unused block-table
entries hold -1 (they are never read).

Workloads (shapes of the decode settings studied on the pages: single query
token per sequence, paged KV, GQA / MLA variants, long and mixed contexts):

  tiny   B 2, Hq 4, Hkv 4, D 64, fp16, bs 16, ctx {17, 40}, 8-block pool
  gqa    B 32, Hq 32, Hkv 8, D 128, bf16, bs 16, ctx ~ U[512, 4096], pool 1.25x
  long   B 4, Hq 32, Hkv 8, D 128, bf16, bs 64, ctx 131072 each, exact pool
  mla    B 64, H 128, latent 576 (V = first 512), bf16, bs 64, ctx ~ U[1024, 8192]
  mixed  B 256, Hq 64, Hkv 8, D 128, bf16, bs 16, ctx log-uniform in [1, 32768]
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class GQAWorkload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str            # "f16" | "bf16"
    block_size: int
    ctx: str              # "fixed:17,40" | "uniform:lo,hi" | "const:n" | "loguniform:lo,hi"
    pool: str             # "fixed:N" | "factor:x"
    seed: int
    scale: Optional[float] = None   # default 1/sqrt(head_dim)
    max_ctx: Optional[int] = None   # capacity bound for the block table (tokens)
    kv_dtype: Optional[str] = None  # None: as dtype; "e4m3": float8 codes + per-tensor scale

    @property
    def kind(self):
        return "gqa"


@dataclass(frozen=True)
class MLAWorkload:
    name: str
    batch: int
    num_heads: int
    kv_dim: int           # latent width (key dims)
    v_dim: int            # value = first v_dim latent dims
    dtype: str
    block_size: int
    ctx: str
    pool: str
    seed: int
    scale: float
    max_ctx: Optional[int] = None

    @property
    def kind(self):
        return "mla"


WORKLOADS = {
    "tiny": GQAWorkload("tiny", 2, 4, 4, 64, "f16", 16, "fixed:17,40", "fixed:8", 1001,
                        max_ctx=48),
    "gqa": GQAWorkload("gqa", 32, 32, 8, 128, "bf16", 16, "uniform:512,4096", "factor:1.25",
                       1002, max_ctx=4096),
    "long": GQAWorkload("long", 4, 32, 8, 128, "bf16", 64, "const:131072", "factor:1.0", 1003,
                        max_ctx=131072),
    "mla": MLAWorkload("mla", 64, 128, 576, 512, "bf16", 64, "uniform:1024,8192", "factor:1.0",
                       1004, scale=1.0 / math.sqrt(192.0), max_ctx=8192),
    "mixed": GQAWorkload("mixed", 256, 64, 8, 128, "bf16", 16, "loguniform:1,32768",
                         "factor:1.0", 1005, max_ctx=32768),
    # the GQA decode workload over a float8 KV cache (E4M3 codes, one scale per
    # tensor): the same shapes and lengths, half the KV bytes
    "gqa_fp8": GQAWorkload("gqa_fp8", 32, 32, 8, 128, "bf16", 16, "uniform:512,4096",
                           "factor:1.25", 1007, max_ctx=4096, kv_dtype="e4m3"),
}

# Float8 KV inputs: N(0,1) values times 2^6 rounded to E4M3 (|x| up to ~6 sigma stays
# below the format's 448), stored as codes; the key / value is code x 2^-6.
KV8_SCALE = 1.0 / 64.0

# Sequence-length scaling sweep (the pages' Flash-Decoding microbenchmark: multi-
# head attention on A100 over sequence lengths 512 to 64k at several batch sizes;
# they give no head count).  Plain reading: 16 query heads of dim 128, bf16,
# block size 16, every sequence at the same length; "mha" gives each query head
# its own KV head, "mqa" shares one KV head among all 16.
SWEEP_CTX = (512, 1024, 2048, 4096, 8192, 16384, 32768, 65536)


def scaling(kind: str, ctx: int, batch: int = 1) -> GQAWorkload:
    hkv = {"mha": 16, "mqa": 1}[kind]
    return GQAWorkload(f"{kind}_{ctx}", batch, 16, hkv, 128, "bf16", 16, f"const:{ctx}",
                       "factor:1.0", 1006, max_ctx=ctx)


TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16}


def get(name: str, **overrides):
    """A named workload, optionally with fields replaced (e.g. batch=4)."""
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def draw_context_lens(spec: str, batch: int, gen: torch.Generator) -> torch.Tensor:
    kind, _, args = spec.partition(":")
    if kind == "fixed":
        vals = [int(x) for x in args.split(",")]
        assert len(vals) == batch, (spec, batch)
        return torch.tensor(vals, dtype=torch.int32)
    if kind == "const":
        return torch.full((batch,), int(args), dtype=torch.int32)
    lo, hi = (int(x) for x in args.split(","))
    if kind == "uniform":
        return torch.randint(lo, hi + 1, (batch,), generator=gen, dtype=torch.int64).to(torch.int32)
    if kind == "loguniform":
        u = torch.rand(batch, generator=gen, dtype=torch.float64)
        x = torch.exp(u * (math.log(hi) - math.log(lo)) + math.log(lo)).floor()
        return x.clamp(lo, hi).to(torch.int32)
    raise ValueError(spec)


def _pool_size(spec: str, needed: int) -> int:
    kind, _, arg = spec.partition(":")
    if kind == "fixed":
        n = int(arg)
        assert n >= needed, (spec, needed)
        return n
    return max(needed, int(math.ceil(float(arg) * needed)))


def build_block_table(context_lens: torch.Tensor, block_size: int, max_blocks: int,
                      pool: int, gen: torch.Generator) -> torch.Tensor:
    """[B, max_blocks] int32: sequence b's logical block j -> physical block id.

    Ids come from one seeded permutation of the pool, handed out in sequence
    order; entries past ceil(ctx/bs) are -1.
    """
    B = context_lens.numel()
    nblk = [(int(c) + block_size - 1) // block_size for c in context_lens.tolist()]
    perm = torch.randperm(pool, generator=gen).to(torch.int32)
    table = torch.full((B, max_blocks), -1, dtype=torch.int32)
    pos = 0
    for b, n in enumerate(nblk):
        assert n <= max_blocks
        table[b, :n] = perm[pos:pos + n]
        pos += n
    return table


def _randn_e4m3(shape, gen, chunk_rows=4096):
    """N(0,1) float32 draws times 1 / KV8_SCALE rounded to E4M3 codes (uint8)."""
    out = torch.empty(shape, dtype=torch.uint8)
    flat = out.view(shape[0], -1)
    for r in range(0, shape[0], chunk_rows):
        rows = min(chunk_rows, shape[0] - r)
        x = torch.randn((rows, flat.shape[1]), generator=gen, dtype=torch.float32) / KV8_SCALE
        flat[r:r + rows] = x.to(torch.float8_e4m3fn).view(torch.uint8)
    return out


def _randn16(shape, dtype, gen, chunk_rows=4096):
    """N(0,1) float32 draws rounded to a 16-bit type, drawn in row chunks."""
    out = torch.empty(shape, dtype=TORCH_DTYPE[dtype])
    flat = out.view(shape[0], -1)
    for r in range(0, shape[0], chunk_rows):
        rows = min(chunk_rows, shape[0] - r)
        flat[r:r + rows] = torch.randn((rows, flat.shape[1]), generator=gen,
                                       dtype=torch.float32).to(out.dtype)
    return out


def make(w, context_lens: Optional[torch.Tensor] = None):
    """Draw the inputs of workload ``w`` (GQA or MLA) on the CPU.

    Returns a dict of CPU tensors plus the scalar fields the call needs.
    """
    gen = torch.Generator().manual_seed(w.seed)
    cl = draw_context_lens(w.ctx, w.batch, gen)
    if context_lens is not None:
        cl = context_lens.to(torch.int32).clone()
    max_ctx = w.max_ctx if w.max_ctx is not None else int(cl.max())
    max_ctx = max(max_ctx, int(cl.max()) if cl.numel() else 0)
    mbs = max(1, (max_ctx + w.block_size - 1) // w.block_size)
    needed = sum((int(c) + w.block_size - 1) // w.block_size for c in cl.tolist())
    nb = _pool_size(w.pool, max(needed, 1))
    table = build_block_table(cl, w.block_size, mbs, nb, gen)
    if w.kind == "gqa":
        q = _randn16((w.batch, w.num_q_heads, w.head_dim), w.dtype, gen)
        kv_shape = (nb, w.num_kv_heads, w.block_size, w.head_dim)
        scale = w.scale if w.scale is not None else 1.0 / math.sqrt(w.head_dim)
        if w.kv_dtype == "e4m3":
            k, v = _randn_e4m3(kv_shape, gen), _randn_e4m3(kv_shape, gen)
            return dict(kind="gqa", q=q, k_cache=k, v_cache=v, block_table=table,
                        context_lens=cl, scale=scale, dtype=w.dtype, kv_dtype="e4m3",
                        k_scale=KV8_SCALE, v_scale=KV8_SCALE, num_blocks=nb,
                        max_blocks_per_seq=mbs)
        k = _randn16(kv_shape, w.dtype, gen)
        v = _randn16(kv_shape, w.dtype, gen)
        return dict(kind="gqa", q=q, k_cache=k, v_cache=v, block_table=table, context_lens=cl,
                    scale=scale, dtype=w.dtype, num_blocks=nb, max_blocks_per_seq=mbs)
    q = _randn16((w.batch, w.num_heads, w.kv_dim), w.dtype, gen)
    lat = _randn16((nb, w.block_size, w.kv_dim), w.dtype, gen)
    return dict(kind="mla", q=q, latent_cache=lat, block_table=table, context_lens=cl,
                scale=w.scale, dtype=w.dtype, v_dim=w.v_dim, num_blocks=nb,
                max_blocks_per_seq=mbs)


@dataclass(frozen=True)
class IndexedWorkload:
    """GQA decode over a per-sequence list of selected token positions."""
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str
    block_size: int
    ctx: int              # context length of every sequence
    top: int              # positions drawn uniformly from [0, ctx - window)
    window: int           # plus the last `window` positions
    seed: int

    @property
    def kind(self):
        return "gqa_indexed"

    @property
    def n_sel(self):
        return self.top + self.window


# Index-list decode (the dense kernel behind sparse top-k attention; the pages'
# DeepSeek-V4 explainer: keep the top 1024 entries plus a 128-token sliding
# window).  The selection is an input: 1024 positions drawn uniformly without
# replacement from [0, ctx - 128), sorted, plus the last 128.  Only blocks that
# hold a selected token are in the pool; every other table entry is -1.
INDEXED = {
    "topk": IndexedWorkload("topk", 32, 32, 8, 128, "bf16", 16, 32768, 1024, 128, 1008),
}


def make_indexed(w: IndexedWorkload, n_sel: Optional[torch.Tensor] = None):
    """Draw the inputs of an index-list workload on the CPU (optionally with fewer
    selected positions per sequence, n_sel[b] <= w.n_sel, keeping the first ones)."""
    gen = torch.Generator().manual_seed(w.seed)
    B, bs = w.batch, w.block_size
    mbs = (w.ctx + bs - 1) // bs
    sel = torch.empty((B, w.n_sel), dtype=torch.int32)
    for b in range(B):
        top = torch.randperm(w.ctx - w.window, generator=gen)[:w.top].sort().values
        win = torch.arange(w.ctx - w.window, w.ctx)
        sel[b] = torch.cat([top, win]).to(torch.int32)
    used = [sorted(set((sel[b] // bs).tolist())) for b in range(B)]
    nb = sum(len(u) for u in used)
    perm = torch.randperm(nb, generator=gen).to(torch.int32)
    table = torch.full((B, mbs), -1, dtype=torch.int32)
    k = 0
    for b in range(B):
        for lb in used[b]:
            table[b, lb] = perm[k]
            k += 1
    q = _randn16((B, w.num_q_heads, w.head_dim), w.dtype, gen)
    kv_shape = (nb, w.num_kv_heads, bs, w.head_dim)
    kc, vc = _randn16(kv_shape, w.dtype, gen), _randn16(kv_shape, w.dtype, gen)
    ns = torch.full((B,), w.n_sel, dtype=torch.int32) if n_sel is None else n_sel.to(torch.int32)
    return dict(kind="gqa_indexed", q=q, k_cache=kc, v_cache=vc, block_table=table,
                token_index=sel, n_sel=ns, context_lens=torch.full((B,), w.ctx, dtype=torch.int32),
                scale=1.0 / math.sqrt(w.head_dim), dtype=w.dtype, num_blocks=nb,
                max_blocks_per_seq=mbs)


def kv_bytes(w, context_lens: torch.Tensor) -> int:
    """Bytes of live KV the operation must read once: every cached element of
    every live token (q, out, block table and scratch excluded).  MLA counts the
    latent once because the value is a prefix of it."""
    tokens = int(context_lens.to(torch.int64).sum())
    if w.kind == "gqa_indexed":        # context_lens here: the selected counts n_sel
        return tokens * w.num_kv_heads * w.head_dim * 2 * 2
    if w.kind == "gqa":
        elem = 1 if w.kv_dtype == "e4m3" else 2
        return tokens * w.num_kv_heads * w.head_dim * 2 * elem
    return tokens * w.kv_dim * 2


def flops(w, context_lens: torch.Tensor) -> int:
    """Multiply-add work of the scores and the value mix, 2 flops per MAC."""
    tokens = int(context_lens.to(torch.int64).sum())
    if w.kind == "gqa":
        return tokens * w.num_q_heads * (w.head_dim + w.head_dim) * 2
    return tokens * w.num_heads * (w.kv_dim + w.v_dim) * 2
