"""CPU checks of the C ABI: the library builds and loads, exports every entry
point include/pa.h declares, and rejects bad arguments on the host before any
CUDA call (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


@pytest.fixture(scope="module")
def lib():
    from paged_split_kv_attention_b200 import _build
    _build.build()
    import paged_split_kv_attention_b200 as pa
    return pa.library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(pa_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("pa_decode", "pa_decode_mla", "pa_workspace_size", "pa_mla_workspace_size",
                 "pa_decode_partition", "pa_decode_merge", "pa_decode_mla_partition",
                 "pa_decode_mla_merge", "pa_decode_fused", "pa_device_status",
                 "pa_status_string"):
        assert want in names, names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in pa.h but not exported"


def test_status_strings(lib):
    import paged_split_kv_attention_b200 as pa
    for s in range(7):
        assert pa.status_string(s)
    assert "unknown" in pa.status_string(99)


def _desc(**kw):
    import paged_split_kv_attention_b200 as pa
    d = dict(batch=4, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
             max_blocks_per_seq=64, num_blocks=300, dtype=pa.PA_BF16, num_partitions=10)
    d.update(kw)
    return pa.PADesc(**d)


def test_workspace_size_is_host_computable(lib):
    import paged_split_kv_attention_b200 as pa
    n = lib.pa_workspace_size(ctypes.byref(_desc()))
    slots = 10 + 4 * 8
    assert n >= slots * 4 * 128 * 4 + slots * 4 * 4 + 5 * 4
    assert lib.pa_workspace_size(ctypes.byref(_desc(num_partitions=20))) > n
    assert lib.pa_workspace_size(None) == 0


@pytest.mark.parametrize("bad,status", [
    (dict(num_q_heads=30), 1),          # Hq not a multiple of Hkv
    (dict(head_dim=96), 2),             # unsupported head dim
    (dict(block_size=8), 2),            # block size not a multiple of 16
    (dict(num_q_heads=8 * 17), 2),      # group of 17 heads
    (dict(batch=-1), 1),
    (dict(num_partitions=-3), 1),
    (dict(dtype=7), 1),
])
def test_invalid_descriptors_are_rejected_before_launch(lib, bad, status):
    d = _desc(**bad)
    z = ctypes.c_void_p(0x1000)
    rc = lib.pa_decode(ctypes.byref(d), z, z, z, z, z, 0.1, z, z, 1 << 30, None)
    assert rc == status
    assert lib.pa_workspace_size(ctypes.byref(d)) == 0


def test_null_pointers_and_small_workspace_are_rejected(lib):
    import paged_split_kv_attention_b200 as pa
    d = _desc()
    z = ctypes.c_void_p(0x1000)
    null = ctypes.c_void_p(0)
    assert lib.pa_decode(ctypes.byref(d), null, z, z, z, z, 0.1, z, z, 1 << 30, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_decode(ctypes.byref(d), z, z, z, z, z, 0.1, z, z, 16, None) == pa.PA_ERR_WORKSPACE
    assert lib.pa_decode(ctypes.byref(d), ctypes.c_void_p(0x1002), z, z, z, z, 0.1, z, z, 1 << 30,
                         None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_decode(ctypes.byref(d), z, z, z, z, z, float("nan"), z, z, 1 << 30,
                         None) == pa.PA_ERR_INVALID_ARG


def test_empty_batch_is_a_no_op(lib):
    d = _desc(batch=0)
    null = ctypes.c_void_p(0)
    assert lib.pa_decode(ctypes.byref(d), null, null, null, null, null, 0.1, null, null, 0, None) == 0


def test_batch_limits(lib):
    import paged_split_kv_attention_b200 as pa
    z = ctypes.c_void_p(0x1000)
    assert lib.pa_workspace_size(ctypes.byref(_desc(batch=4096))) > 0
    big = _desc(batch=4097)
    assert lib.pa_workspace_size(ctypes.byref(big)) == 0
    assert lib.pa_decode(ctypes.byref(big), z, z, z, z, z, 0.1, z, z, 1 << 30, None) == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_decode_fused(ctypes.byref(big), z, z, z, z, z, 0.1, z, z, 1 << 30,
                               None) == pa.PA_ERR_UNSUPPORTED

    def mla(batch):
        return pa.PAMLADesc(batch, 128, 576, 512, 64, 32, 4096, pa.PA_BF16, 10)
    assert lib.pa_mla_workspace_size(ctypes.byref(mla(32768))) > 0
    assert lib.pa_mla_workspace_size(ctypes.byref(mla(32769))) == 0


def test_fused_entry_point_rejects_what_pa_decode_rejects(lib):
    z = ctypes.c_void_p(0x1000)
    for bad in (dict(num_q_heads=30), dict(head_dim=96), dict(batch=-1)):
        d = _desc(**bad)
        assert (lib.pa_decode_fused(ctypes.byref(d), z, z, z, z, z, 0.1, z, z, 1 << 30, None) ==
                lib.pa_decode(ctypes.byref(d), z, z, z, z, z, 0.1, z, z, 1 << 30, None) != 0)


def test_index_list_size_limit(lib):
    import paged_split_kv_attention_b200 as pa
    z = ctypes.c_void_p(0x1000)
    d = _desc(batch=4096, num_kv_heads=8, num_q_heads=32)
    huge = (1 << 31) // (4096 * 8) * 16
    assert lib.pa_decode_indexed(ctypes.byref(d), z, z, z, z, z, huge, z, 0.1, z, z, 1 << 30,
                                 None) == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_decode_indexed(ctypes.byref(d), z, z, z, z, z, 0, z, 0.1, z, z, 1 << 30,
                                 None) == pa.PA_ERR_INVALID_ARG


def test_float8_entry_point_validation(lib):
    import paged_split_kv_attention_b200 as pa
    z = ctypes.c_void_p(0x1000)
    d = _desc()
    for ks, vs in ((float("nan"), 1.0), (1.0, float("inf")), (float("-inf"), 1.0)):
        assert lib.pa_decode_kv_e4m3(ctypes.byref(d), z, z, z, z, z, 0.1, ks, vs, z, z, 1 << 30,
                                     None) == pa.PA_ERR_INVALID_ARG
    d64 = _desc(head_dim=64)
    assert lib.pa_decode_kv_e4m3(ctypes.byref(d64), z, z, z, z, z, 0.1, 1.0, 1.0, z, z, 1 << 30,
                                 None) == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_decode_indexed(ctypes.byref(d64), z, z, z, z, z, 16, z, 0.1, z, z, 1 << 30,
                                 None) == pa.PA_ERR_UNSUPPORTED
    # the partition / merge forms validate alike
    for name in ("pa_decode_kv_e4m3_partition", "pa_decode_kv_e4m3_merge"):
        assert getattr(lib, name)(ctypes.byref(d), z, z, z, z, z, 0.1, float("nan"), 1.0, z, z,
                                  1 << 30, None) == pa.PA_ERR_INVALID_ARG
    for name in ("pa_decode_indexed_partition", "pa_decode_indexed_merge"):
        assert getattr(lib, name)(ctypes.byref(d), z, z, z, z, z, 0, z, 0.1, z, z, 1 << 30,
                                  None) == pa.PA_ERR_INVALID_ARG


def test_header_is_plain_c_and_links(lib, tmp_path):
    # the boundary is a C ABI: the header compiles as C (and C++), and a C program
    # links against the library and calls a host-side entry point
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "use_pa.c"
    src.write_text(
        '#include "pa.h"\n#include <stdio.h>\n'
        "int main(void) {\n"
        "  pa_desc d = {4, 32, 8, 128, 16, 64, 300, PA_BF16, 10};\n"
        "  size_t n = pa_workspace_size(&d);\n"
        '  printf("%zu %s\\n", n, pa_status_string(PA_ERR_UNSUPPORTED));\n'
        "  return n > 0 ? 0 : 1;\n}\n")
    libdir = os.path.join(ROOT, "paged_split_kv_attention_b200")
    exe = tmp_path / "use_pa"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lpa_b200", "-Wl,-rpath," + libdir, "-o", str(exe)],
                   check=True, capture_output=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "unsupported" in r.stdout
    subprocess.run(["g++", "-std=c++17", "-fsyntax-only", "-Wall", "-Werror", "-x", "c++",
                    os.path.join(ROOT, "include", "pa.h")], check=True, capture_output=True)
