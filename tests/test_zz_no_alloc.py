"""GPU test of pa_decode_static, the entry point for callers that cannot allocate.

Some callers have no way to provide device scratch (a host runtime that owns all
device memory, a serving loop that must not call cudaMalloc because it can
synchronise the device, a plain C program without a caching allocator).
pa_decode_static runs the same decode as pa_decode but keeps its scratch in a
fixed 16 MiB buffer inside the library.  This test calls it through the C ABI
twice in a row and checks each result against pa_decode (which uses a caller
workspace): both run the same kernels with the same pieces, so the outputs must
be bitwise equal, and the tiny workload is also checked against the float64
oracle with the tolerance of the other parity tests.  After a first call has
loaded everything, a further call must leave the device's free memory and
torch's allocator untouched.  The file is collected last, and it passes alone
or after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2


def _lib():
    import paged_split_kv_attention_b200 as pa
    lib = pa.library()
    lib.pa_decode_static.argtypes = [ctypes.POINTER(pa.PADesc)] + [ctypes.c_void_p] * 5 + \
        [ctypes.c_float] + [ctypes.c_void_p] * 2
    lib.pa_decode_static.restype = ctypes.c_int
    return pa, lib


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("name,overrides", [("gqa", dict(batch=8)), ("mixed", dict(batch=24)),
                                            ("tiny", {})])
def test_static_scratch_matches_workspace_call_twice(cuda_device, name, overrides):
    pa, lib = _lib()
    inp = workloads.make(workloads.get(name, **overrides))
    d = {k: (v.to(cuda_device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    ref = pa.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["context_lens"],
                    inp["scale"])
    torch.cuda.synchronize()
    desc = pa.gqa_desc(d["q"], d["k_cache"], d["block_table"])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    outs = [torch.full_like(d["q"], float("nan")) for _ in range(3)]

    def call(out):
        return lib.pa_decode_static(ctypes.byref(desc), _ptr(d["q"]), _ptr(d["k_cache"]),
                                    _ptr(d["v_cache"]), _ptr(d["block_table"]),
                                    _ptr(d["context_lens"]), ctypes.c_float(inp["scale"]),
                                    _ptr(out), stream)

    # two calls in a row, each compared with the workspace call
    for out in outs[:2]:
        rc = call(out)
        assert rc == pa.PA_OK, pa.status_string(rc)
        torch.cuda.synchronize()
        assert pa.device_status() == pa.PA_OK
        assert torch.equal(out, ref)

    # a third call allocates nothing: device free memory and torch's allocator
    # are unchanged across it (the first calls loaded the module and looked up
    # the buffer's address)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    reserved0 = torch.cuda.memory_reserved()
    rc = call(outs[2])
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert rc == pa.PA_OK, pa.status_string(rc)
    assert free1 >= free0
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.memory_reserved() == reserved0
    assert torch.equal(outs[2], ref)

    if name == "tiny":
        exp = oracle.decode(_u16(inp["q"]), _u16(inp["k_cache"]), _u16(inp["v_cache"]),
                            inp["block_table"].numpy(), inp["context_lens"].numpy(),
                            inp["scale"], inp["dtype"])
        g = outs[0].float().cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all()
        assert (np.abs(g - exp) <= ATOL + RTOL * np.abs(exp)).all()


def test_call_larger_than_static_scratch_is_rejected(cuda_device):
    pa, lib = _lib()
    # 4096 sequences x 8 kv heads x 16 heads per group: scratch far above 16 MiB
    desc = pa.PADesc(4096, 128, 8, 128, 16, 64, 100000, pa.PA_BF16, 0)
    dummy = ctypes.c_void_p(256)        # never dereferenced: rejected before any launch
    rc = lib.pa_decode_static(ctypes.byref(desc), dummy, dummy, dummy, dummy, dummy,
                              ctypes.c_float(0.1), dummy, None)
    assert rc == pa.PA_ERR_TOO_LARGE
    assert "static" in pa.status_string(rc)
