"""B200-native paged split-KV decode attention.

Thin Python binding of ``libpa_b200.so`` (C ABI declared in ``include/pa.h``).
This module only marshals arguments: it checks tensor shapes/dtypes, takes raw
device pointers from torch tensors, allocates the output and the scratch
workspace with torch when the caller does not pass them, and calls the library
on the current torch CUDA stream.  Every step of the computation runs in the
library's CUDA kernels; there is no other code path.  If the shared library is
missing, every call raises -- there is no fallback.

    out = decode(q, k_cache, v_cache, block_table, context_lens, scale)
    out = decode_mla(q, latent_cache, block_table, context_lens, scale, v_dim=512)
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa_b200.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_CUDA = 0, 1, 2, 3
PA_ERR_BAD_BLOCK_ID, PA_ERR_TIMEOUT, PA_ERR_WORKSPACE = 4, 5, 6
PA_F16, PA_BF16 = 0, 1

_DTYPES = {torch.float16: PA_F16, torch.bfloat16: PA_BF16}


class PADesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("num_q_heads", ctypes.c_int),
                ("num_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("block_size", ctypes.c_int), ("max_blocks_per_seq", ctypes.c_int),
                ("num_blocks", ctypes.c_int), ("dtype", ctypes.c_int),
                ("num_partitions", ctypes.c_int)]


class PAMLADesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("num_heads", ctypes.c_int), ("kv_dim", ctypes.c_int),
                ("v_dim", ctypes.c_int), ("block_size", ctypes.c_int),
                ("max_blocks_per_seq", ctypes.c_int), ("num_blocks", ctypes.c_int),
                ("dtype", ctypes.c_int), ("num_partitions", ctypes.c_int)]


class PAError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})" if what
                         else f"{status_string(status)} (status {status})")


_lib = None
_lock = threading.Lock()


def library() -> ctypes.CDLL:
    """The loaded C library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; "
                    f"g.build()'` (nvcc, sm_100a). There is no fallback path.")
            lib = ctypes.CDLL(LIB_PATH)
            vp, sz, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float
            gqa = [ctypes.POINTER(PADesc), vp, vp, vp, vp, vp, f32, vp, vp, sz, vp]
            mla = [ctypes.POINTER(PAMLADesc), vp, vp, vp, vp, f32, vp, vp, sz, vp]
            for name in ("pa_decode", "pa_decode_partition", "pa_decode_merge", "pa_decode_fused"):
                getattr(lib, name).argtypes = gqa
                getattr(lib, name).restype = ctypes.c_int
            for name in ("pa_decode_mla", "pa_decode_mla_partition", "pa_decode_mla_merge"):
                getattr(lib, name).argtypes = mla
                getattr(lib, name).restype = ctypes.c_int
            for name in ("pa_decode_kv_e4m3", "pa_decode_kv_e4m3_partition",
                         "pa_decode_kv_e4m3_merge"):
                getattr(lib, name).argtypes = [ctypes.POINTER(PADesc), vp, vp, vp, vp, vp, f32, f32,
                                               f32, vp, vp, sz, vp]
                getattr(lib, name).restype = ctypes.c_int
            for name in ("pa_decode_indexed", "pa_decode_indexed_partition",
                         "pa_decode_indexed_merge"):
                getattr(lib, name).argtypes = [ctypes.POINTER(PADesc), vp, vp, vp, vp, vp,
                                               ctypes.c_int, vp, f32, vp, vp, sz, vp]
                getattr(lib, name).restype = ctypes.c_int
            lib.pa_workspace_size.argtypes = [ctypes.POINTER(PADesc)]
            lib.pa_workspace_size.restype = sz
            lib.pa_mla_workspace_size.argtypes = [ctypes.POINTER(PAMLADesc)]
            lib.pa_mla_workspace_size.restype = sz
            lib.pa_default_partitions.argtypes = [ctypes.c_int, ctypes.c_int]
            lib.pa_default_partitions.restype = ctypes.c_int
            lib.pa_device_status.argtypes = [vp, ctypes.c_int]
            lib.pa_device_status.restype = ctypes.c_int
            lib.pa_test_inject_stall.argtypes = [ctypes.c_int]
            lib.pa_test_inject_stall.restype = None
            lib.pa_status_string.argtypes = [ctypes.c_int]
            lib.pa_status_string.restype = ctypes.c_char_p
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return library().pa_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != PA_OK:
        raise PAError(status, what)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream_ptr(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def gqa_desc(q, k_cache, block_table, num_partitions=0) -> PADesc:
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D:
        raise ValueError(f"head_dim mismatch: q {D}, cache {D2}")
    if q.dtype not in _DTYPES:
        raise TypeError(f"dtype {q.dtype} not supported (fp16/bf16)")
    return PADesc(B, Hq, Hkv, D, bs, block_table.shape[1], NB, _DTYPES[q.dtype],
                  int(num_partitions))


def mla_desc(q, latent_cache, block_table, v_dim, num_partitions=0) -> PAMLADesc:
    B, H, Dk = q.shape
    NB, bs, Dk2 = latent_cache.shape
    if Dk2 != Dk:
        raise ValueError(f"kv_dim mismatch: q {Dk}, cache {Dk2}")
    if q.dtype not in _DTYPES:
        raise TypeError(f"dtype {q.dtype} not supported (fp16/bf16)")
    return PAMLADesc(B, H, Dk, int(v_dim), bs, block_table.shape[1], NB, _DTYPES[q.dtype],
                     int(num_partitions))


def workspace_size(desc) -> int:
    lib = library()
    if isinstance(desc, PADesc):
        return int(lib.pa_workspace_size(ctypes.byref(desc)))
    return int(lib.pa_mla_workspace_size(ctypes.byref(desc)))


def default_partitions(kind: str = "gqa", head_dim: int = 128) -> int:
    """kind: "gqa", "mla", "gqa_fp8" (float8 KV cache) or "gqa_indexed" (index list)."""
    code = {"gqa": 0, "mla": 1, "gqa_fp8": 2, "gqa_indexed": 3}[kind]
    return int(library().pa_default_partitions(code, head_dim))


def _require(t, name, dtype=None, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def _workspace(nbytes, device, workspace):
    if workspace is None:
        return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    if workspace.numel() * workspace.element_size() < nbytes:
        raise PAError(PA_ERR_WORKSPACE, "workspace")
    return workspace


_PASSES = {"both": "pa_decode", "partition": "pa_decode_partition", "merge": "pa_decode_merge",
           "fused": "pa_decode_fused"}
_MLA_PASSES = {"both": "pa_decode_mla", "partition": "pa_decode_mla_partition",
               "merge": "pa_decode_mla_merge"}


def decode(q, k_cache, v_cache, block_table, context_lens, scale, out=None, workspace=None,
           num_partitions=0, stream=None, passes="both"):
    """Paged GQA/MHA/MQA decode attention, one query token per sequence.

    q [B, Hq, D]; k_cache, v_cache [num_blocks, Hkv, block_size, D] (fp16/bf16);
    block_table [B, max_blocks_per_seq] int32; context_lens [B] int32.
    Returns out [B, Hq, D] in q's dtype.  Asynchronous on the current stream.
    passes="partition" / "merge" run one of the two kernels (merge must follow
    partition with the same arguments and workspace); passes="fused" is the
    single-launch form (pa_decode_fused: the last piece of each split sequence
    and kv head merges it).
    """
    _require(q, "q", ndim=3)
    _require(k_cache, "k_cache", q.dtype, 4)
    _require(v_cache, "v_cache", q.dtype, 4)
    _require(block_table, "block_table", torch.int32, 2)
    _require(context_lens, "context_lens", torch.int32, 1)
    if v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache shapes differ")
    desc = gqa_desc(q, k_cache, block_table, num_partitions)
    if out is None:
        out = torch.empty_like(q)
    else:
        _require(out, "out", q.dtype, 3)
    ws_bytes = workspace_size(desc)
    if ws_bytes == 0:
        raise PAError(PA_ERR_INVALID_ARG if torch.cuda.is_available() else PA_ERR_CUDA,
                      "pa_workspace_size")
    ws = _workspace(ws_bytes, q.device, workspace)
    fn = getattr(library(), _PASSES[passes])
    _check(fn(ctypes.byref(desc), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
              _ptr(context_lens), float(scale), _ptr(out), _ptr(ws),
              ws.numel() * ws.element_size(), _stream_ptr(stream)), _PASSES[passes])
    return out


_KV8_PASSES = {"both": "pa_decode_kv_e4m3", "partition": "pa_decode_kv_e4m3_partition",
               "merge": "pa_decode_kv_e4m3_merge"}
_IDX_PASSES = {"both": "pa_decode_indexed", "partition": "pa_decode_indexed_partition",
               "merge": "pa_decode_indexed_merge"}


def decode_kv8(q, k_cache, v_cache, block_table, context_lens, scale, k_scale, v_scale,
               out=None, workspace=None, num_partitions=0, stream=None, passes="both"):
    """pa_decode_kv_e4m3: paged GQA/MHA/MQA decode over a float8 KV cache.

    k_cache, v_cache [num_blocks, Hkv, block_size, 128] uint8 holding E4M3 codes;
    the key is code * k_scale and the value code * v_scale.  q [B, Hq, 128] fp16 or
    bf16 (bf16 within the fp16 range).  Returns out [B, Hq, 128] in q's dtype.
    passes="partition" / "merge" run one of the two kernels, as for decode().
    """
    _require(q, "q", ndim=3)
    _require(k_cache, "k_cache", torch.uint8, 4)
    _require(v_cache, "v_cache", torch.uint8, 4)
    _require(block_table, "block_table", torch.int32, 2)
    _require(context_lens, "context_lens", torch.int32, 1)
    if v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache shapes differ")
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D:
        raise ValueError(f"head_dim mismatch: q {D}, cache {D2}")
    if q.dtype not in _DTYPES:
        raise TypeError(f"dtype {q.dtype} not supported (fp16/bf16)")
    desc = PADesc(B, Hq, Hkv, D, bs, block_table.shape[1], NB, _DTYPES[q.dtype],
                  int(num_partitions))
    if out is None:
        out = torch.empty_like(q)
    else:
        _require(out, "out", q.dtype, 3)
    ws_bytes = workspace_size(desc)
    if ws_bytes == 0:
        raise PAError(PA_ERR_UNSUPPORTED, "pa_workspace_size")
    ws = _workspace(ws_bytes, q.device, workspace)
    fn = _KV8_PASSES[passes]
    _check(getattr(library(), fn)(ctypes.byref(desc), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(block_table), _ptr(context_lens), float(scale),
                                  float(k_scale), float(v_scale), _ptr(out), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream_ptr(stream)), fn)
    return out


def decode_indexed(q, k_cache, v_cache, block_table, token_index, n_sel, scale, out=None,
                   workspace=None, num_partitions=0, stream=None, passes="both"):
    """pa_decode_indexed: each sequence attends over a list of its token positions.

    token_index [B, max_sel] int32 positions; n_sel [B] int32 counts (entries past
    n_sel[b] are never read).  Caches and q as decode() (head_dim 128).
    passes="partition" / "merge" run one of the two kernels, as for decode().
    """
    _require(q, "q", ndim=3)
    _require(k_cache, "k_cache", q.dtype, 4)
    _require(v_cache, "v_cache", q.dtype, 4)
    _require(block_table, "block_table", torch.int32, 2)
    _require(token_index, "token_index", torch.int32, 2)
    _require(n_sel, "n_sel", torch.int32, 1)
    if v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache shapes differ")
    desc = gqa_desc(q, k_cache, block_table, num_partitions)
    if out is None:
        out = torch.empty_like(q)
    else:
        _require(out, "out", q.dtype, 3)
    ws_bytes = workspace_size(desc)
    if ws_bytes == 0:
        raise PAError(PA_ERR_UNSUPPORTED, "pa_workspace_size")
    ws = _workspace(ws_bytes, q.device, workspace)
    fn = _IDX_PASSES[passes]
    _check(getattr(library(), fn)(ctypes.byref(desc), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(block_table), _ptr(token_index),
                                  int(token_index.shape[1]), _ptr(n_sel), float(scale),
                                  _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream_ptr(stream)), fn)
    return out


def decode_mla(q, latent_cache, block_table, context_lens, scale, v_dim=512, out=None,
               workspace=None, num_partitions=0, stream=None, passes="both"):
    """MLA absorbed decode: every head reads one shared latent row per token.

    q [B, H, kv_dim]; latent_cache [num_blocks, block_size, kv_dim]; the value is
    the first v_dim latent dims.  Returns out [B, H, v_dim].
    """
    _require(q, "q", ndim=3)
    _require(latent_cache, "latent_cache", q.dtype, 3)
    _require(block_table, "block_table", torch.int32, 2)
    _require(context_lens, "context_lens", torch.int32, 1)
    desc = mla_desc(q, latent_cache, block_table, v_dim, num_partitions)
    if out is None:
        out = torch.empty((q.shape[0], q.shape[1], v_dim), dtype=q.dtype, device=q.device)
    else:
        _require(out, "out", q.dtype, 3)
    ws_bytes = workspace_size(desc)
    if ws_bytes == 0:
        raise PAError(PA_ERR_UNSUPPORTED, "pa_mla_workspace_size")
    ws = _workspace(ws_bytes, q.device, workspace)
    fn = getattr(library(), _MLA_PASSES[passes])
    _check(fn(ctypes.byref(desc), _ptr(q), _ptr(latent_cache), _ptr(block_table),
              _ptr(context_lens), float(scale), _ptr(out), _ptr(ws),
              ws.numel() * ws.element_size(), _stream_ptr(stream)), _MLA_PASSES[passes])
    return out


def inject_stall_for_testing(enable: bool) -> None:
    """Test hook (pa_test_inject_stall): while enabled, GQA partition launches
    take their bounded-wait timeout path and report PA_ERR_TIMEOUT."""
    library().pa_test_inject_stall(1 if enable else 0)


def device_status(reset: bool = True, stream=None) -> int:
    """Synchronise the stream and return (then clear) the first error the kernels
    recorded on the current device (PA_OK if none)."""
    return int(library().pa_device_status(_stream_ptr(stream), 1 if reset else 0))


PA_ERR_TOO_LARGE = 7


def decode_static(q, k_cache, v_cache, block_table, context_lens, scale, out=None,
                  num_partitions=0, stream=None):
    """pa_decode_static: the same decode with the library's fixed 16 MiB device
    scratch instead of a caller workspace, for callers that cannot allocate
    device memory (the output is still the caller's).  Calls that overlap on the
    GPU share that buffer and must be serialised."""
    lib = library()
    fn = lib.pa_decode_static
    fn.argtypes = [ctypes.POINTER(PADesc)] + [ctypes.c_void_p] * 5 + [ctypes.c_float] + \
        [ctypes.c_void_p] * 2
    fn.restype = ctypes.c_int
    _require(q, "q", ndim=3)
    _require(k_cache, "k_cache", q.dtype, 4)
    _require(v_cache, "v_cache", q.dtype, 4)
    _require(block_table, "block_table", torch.int32, 2)
    _require(context_lens, "context_lens", torch.int32, 1)
    desc = gqa_desc(q, k_cache, block_table, num_partitions)
    if out is None:
        out = torch.empty_like(q)
    _check(fn(ctypes.byref(desc), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
              _ptr(context_lens), float(scale), _ptr(out), _stream_ptr(stream)),
           "pa_decode_static")
    return out
