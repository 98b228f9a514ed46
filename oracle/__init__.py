"""float64 CPU oracle for paged split-KV decode attention.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference leg may import this package; the product path
(``paged_split_kv_attention_b200``) never does, and the two share no code.

The arithmetic lives in ``pa_oracle.c`` (plain C, IEEE double, optional OpenMP
over (sequence, head) pairs).  This module only compiles it with gcc when the
shared object is missing or older than the source, and marshals numpy arrays
through ctypes.  Inputs are the raw 16-bit patterns of the fp16/bf16 tensors
the GPU path consumes, so both sides see bit-identical values.

Functions and the passages they follow (the C file states the same):
  decode        -- paged softmax(q K^T * scale) V, the definition (pages
                   "wenku.it search: paged attention" and "...: Multi-head Latent
                   Attention (MLA)", Transformer-introduction snippets; page
                   "bjpcjp.github.io: llms-attention", softmax-attention abstract)
  decode_split  -- the same through per-split softmax + log-sum-exp merge (page
                   "cidian.kuaisou.com: flash decoding ++", three-step snippets)
  decode_mla    -- shared-latent absorbed decode, V = first Dv latent dims (page
                   "wenku.it search: Multi-head Latent Attention (MLA)",
                   DeepSeek-V2 abstract)
  f16_to_f64 / bf16_to_f64 -- exact decoding of the 16-bit input formats
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB = os.path.join(_HERE, "libpa_oracle.so")
_lock = threading.Lock()
_lib = None

F16, BF16 = 0, 1
_STATUS = {0: "ok", 1: "bad argument", 2: "block id out of range", 3: "out of memory"}


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into libpa_oracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            p16 = ctypes.POINTER(ctypes.c_uint16)
            p32 = ctypes.POINTER(ctypes.c_int32)
            pf64 = ctypes.POINTER(ctypes.c_double)
            i, d = ctypes.c_int, ctypes.c_double
            lib.pa_oracle_decode.argtypes = [i] * 8 + [p16, p16, p16, p32, p32, d, p32, i, pf64, i]
            lib.pa_oracle_decode_split.argtypes = [i] * 8 + [p16, p16, p16, p32, p32, d, i, pf64, i]
            lib.pa_oracle_decode_mla.argtypes = [i] * 8 + [p16, p16, p32, p32, d, p32, i, pf64, i]
            p8 = ctypes.POINTER(ctypes.c_uint8)
            lib.pa_oracle_decode_kv8.argtypes = [i] * 8 + [p16, p8, p8, d, d, p32, p32, d, p32, i,
                                                           pf64, i]
            lib.pa_oracle_decode_indexed.argtypes = [i] * 8 + [p16, p16, p16, p32, p32, i, p32, d,
                                                               p32, i, pf64, i]
            for f in (lib.pa_oracle_decode, lib.pa_oracle_decode_split, lib.pa_oracle_decode_mla,
                      lib.pa_oracle_decode_kv8, lib.pa_oracle_decode_indexed):
                f.restype = ctypes.c_int
            lib.pa_oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
            lib.pa_oracle_f16_to_f64.restype = ctypes.c_double
            lib.pa_oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
            lib.pa_oracle_bf16_to_f64.restype = ctypes.c_double
            lib.pa_oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
            lib.pa_oracle_e4m3_to_f64.restype = ctypes.c_double
            lib.pa_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError(f"expected raw 16-bit patterns (uint16 or float16), got {a.dtype}")
    return a


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _ptr(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _check(rc):
    if rc != 0:
        raise RuntimeError(f"oracle failed: {_STATUS.get(rc, rc)}")


def _dtype_code(dtype: str) -> int:
    return {"f16": F16, "fp16": F16, "float16": F16, "bf16": BF16, "bfloat16": BF16}[dtype]


def max_threads() -> int:
    return _load().pa_oracle_max_threads()


def f16_to_f64(bits: int) -> float:
    return _load().pa_oracle_f16_to_f64(bits)


def bf16_to_f64(bits: int) -> float:
    return _load().pa_oracle_bf16_to_f64(bits)


def decode(q, k_cache, v_cache, block_table, context_lens, scale, dtype, pairs=None,
           nthreads=0):
    """Paged GQA decode in float64.

    q [B,Hq,D], k_cache/v_cache [NB,Hkv,bs,D] (raw uint16 bits), block_table
    [B,MBS] int32, context_lens [B] int32.  Returns float64 [B,Hq,D], or
    [len(pairs), D] when a list of (b, h) pairs is given.
    """
    lib = _load()
    q, k, v = _u16(q), _u16(k_cache), _u16(v_cache)
    bt, cl = _i32(block_table), _i32(context_lens)
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k.shape
    assert D2 == D and v.shape == k.shape and bt.shape[0] == B and cl.shape == (B,)
    mbs = bt.shape[1]
    if pairs is None:
        out = np.empty((B, Hq, D), np.float64)
        pp, npairs = None, 0
    else:
        pp = _i32(pairs).reshape(-1, 2)
        npairs = pp.shape[0]
        out = np.empty((npairs, D), np.float64)
    rc = lib.pa_oracle_decode(B, Hq, Hkv, D, bs, mbs, NB, _dtype_code(dtype),
                              _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
                              _ptr(v, ctypes.c_uint16), _ptr(bt, ctypes.c_int32),
                              _ptr(cl, ctypes.c_int32), float(scale),
                              None if pp is None else _ptr(pp, ctypes.c_int32), npairs,
                              _ptr(out, ctypes.c_double), int(nthreads))
    _check(rc)
    return out


def e4m3_to_f64(code: int) -> float:
    return _load().pa_oracle_e4m3_to_f64(code)


def decode_kv8(q, k_cache, v_cache, k_scale, v_scale, block_table, context_lens, scale, dtype,
               pairs=None, nthreads=0):
    """Paged GQA decode in float64 over a float8 (E4M3) KV cache.

    q [B,Hq,D] raw 16-bit of `dtype`; k_cache/v_cache [NB,Hkv,bs,D] uint8 E4M3 codes;
    key = code * k_scale, value = code * v_scale.  Returns float64 [B,Hq,D], or
    [len(pairs), D] when a list of (b, h) pairs is given.
    """
    lib = _load()
    q = _u16(q)
    k = np.ascontiguousarray(k_cache, dtype=np.uint8)
    v = np.ascontiguousarray(v_cache, dtype=np.uint8)
    bt, cl = _i32(block_table), _i32(context_lens)
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k.shape
    assert D2 == D and v.shape == k.shape and bt.shape[0] == B and cl.shape == (B,)
    if pairs is None:
        out = np.empty((B, Hq, D), np.float64)
        pp, npairs = None, 0
    else:
        pp = _i32(pairs).reshape(-1, 2)
        npairs = pp.shape[0]
        out = np.empty((npairs, D), np.float64)
    rc = lib.pa_oracle_decode_kv8(B, Hq, Hkv, D, bs, bt.shape[1], NB, _dtype_code(dtype),
                                  _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint8),
                                  _ptr(v, ctypes.c_uint8), float(k_scale), float(v_scale),
                                  _ptr(bt, ctypes.c_int32), _ptr(cl, ctypes.c_int32), float(scale),
                                  None if pp is None else _ptr(pp, ctypes.c_int32), npairs,
                                  _ptr(out, ctypes.c_double), int(nthreads))
    _check(rc)
    return out


def decode_indexed(q, k_cache, v_cache, block_table, token_index, n_sel, scale, dtype,
                   pairs=None, nthreads=0):
    """Paged GQA decode over a given list of token positions per sequence.

    token_index [B, max_sel] int32 positions (block block_table[b][pos // bs], row
    pos % bs); n_sel [B] int32 counts.  Other arguments as decode().  Returns
    float64 [B,Hq,D] (or [len(pairs), D]).
    """
    lib = _load()
    q, k, v = _u16(q), _u16(k_cache), _u16(v_cache)
    bt, ti, ns = _i32(block_table), _i32(token_index), _i32(n_sel)
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k.shape
    assert D2 == D and v.shape == k.shape and bt.shape[0] == B and ti.shape[0] == B
    if pairs is None:
        out = np.empty((B, Hq, D), np.float64)
        pp, npairs = None, 0
    else:
        pp = _i32(pairs).reshape(-1, 2)
        npairs = pp.shape[0]
        out = np.empty((npairs, D), np.float64)
    rc = lib.pa_oracle_decode_indexed(B, Hq, Hkv, D, bs, bt.shape[1], NB, _dtype_code(dtype),
                                      _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
                                      _ptr(v, ctypes.c_uint16), _ptr(bt, ctypes.c_int32),
                                      _ptr(ti, ctypes.c_int32), ti.shape[1],
                                      _ptr(ns, ctypes.c_int32), float(scale),
                                      None if pp is None else _ptr(pp, ctypes.c_int32), npairs,
                                      _ptr(out, ctypes.c_double), int(nthreads))
    _check(rc)
    return out


def decode_split(q, k_cache, v_cache, block_table, context_lens, scale, dtype, split_len,
                 nthreads=0):
    """The same GQA decode computed as per-split softmax + log-sum-exp merge."""
    lib = _load()
    q, k, v = _u16(q), _u16(k_cache), _u16(v_cache)
    bt, cl = _i32(block_table), _i32(context_lens)
    B, Hq, D = q.shape
    NB, Hkv, bs, _ = k.shape
    out = np.empty((B, Hq, D), np.float64)
    rc = lib.pa_oracle_decode_split(B, Hq, Hkv, D, bs, bt.shape[1], NB, _dtype_code(dtype),
                                    _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
                                    _ptr(v, ctypes.c_uint16), _ptr(bt, ctypes.c_int32),
                                    _ptr(cl, ctypes.c_int32), float(scale), int(split_len),
                                    _ptr(out, ctypes.c_double), int(nthreads))
    _check(rc)
    return out


def decode_mla(q, latent_cache, block_table, context_lens, scale, dtype, v_dim, pairs=None,
               nthreads=0):
    """Shared-latent absorbed decode in float64.

    q [B,H,Dk], latent_cache [NB,bs,Dk] (raw uint16 bits); the value is the first
    v_dim latent dims.  Returns float64 [B,H,v_dim] (or [len(pairs), v_dim]).
    """
    lib = _load()
    q, lat = _u16(q), _u16(latent_cache)
    bt, cl = _i32(block_table), _i32(context_lens)
    B, H, Dk = q.shape
    NB, bs, Dk2 = lat.shape
    assert Dk2 == Dk and bt.shape[0] == B and cl.shape == (B,)
    if pairs is None:
        out = np.empty((B, H, v_dim), np.float64)
        pp, npairs = None, 0
    else:
        pp = _i32(pairs).reshape(-1, 2)
        npairs = pp.shape[0]
        out = np.empty((npairs, v_dim), np.float64)
    rc = lib.pa_oracle_decode_mla(B, H, Dk, int(v_dim), bs, bt.shape[1], NB, _dtype_code(dtype),
                                  _ptr(q, ctypes.c_uint16), _ptr(lat, ctypes.c_uint16),
                                  _ptr(bt, ctypes.c_int32), _ptr(cl, ctypes.c_int32),
                                  float(scale), None if pp is None else _ptr(pp, ctypes.c_int32),
                                  npairs, _ptr(out, ctypes.c_double), int(nthreads))
    _check(rc)
    return out
