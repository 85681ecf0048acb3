"""The C ABI library loads without a GPU, exports every symbol include/pa.h
declares, and rejects bad arguments before touching the device."""

import ctypes
import os
import re
import subprocess

import pytest

import paged_kv_cache_354_b200 as pk

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "pa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"^(?:const\s+)?\w+\*?\s+\**(pa_\w+)\s*\(", text, flags=re.M))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("pa_reshape_and_cache", "pa_copy_blocks", "pa_decode", "pa_decode_workspace_size",
                     "pa_alloc_create", "pa_alloc_append", "pa_alloc_fork", "pa_alloc_free_seq"):
        assert required in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", pk.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = declared_functions() - exported
    assert not missing, missing
    for name in declared_functions():
        assert hasattr(pk.lib, name)


def test_binding_covers_the_header():
    assert set(pk._SIGNATURES) == declared_functions()


def test_version():
    assert pk.pa_version() >= 100


def test_invalid_arguments_fail_before_launch():
    lib = pk.lib
    # head_dim not a multiple of 8
    assert lib.pa_reshape_and_cache(None, None, None, None, 4, 8, 2, 16, 7, None) == pk.PA_ERR_INVALID
    assert "multiple of 8" in lib.pa_last_error_string().decode()
    # zero tokens / pairs are no-ops even with NULL pointers
    assert lib.pa_reshape_and_cache(None, None, None, None, 0, 8, 2, 16, 64, None) == pk.PA_OK
    assert lib.pa_copy_blocks(None, None, 0, 8, 2, 16, 64, None) == pk.PA_OK
    # NULL pointers with work to do
    assert lib.pa_copy_blocks(None, None, 3, 8, 2, 16, 64, None) == pk.PA_ERR_INVALID
    nb = ctypes.c_size_t()
    parts = ctypes.c_int()
    # unsupported head_dim / block size / group; bad group divisibility
    assert lib.pa_decode_workspace_size(4, 8, 2, 96, 16, 100, ctypes.byref(nb), ctypes.byref(parts)) == \
        pk.PA_ERR_UNSUPPORTED
    assert lib.pa_decode_workspace_size(4, 8, 2, 128, 8, 100, ctypes.byref(nb), ctypes.byref(parts)) == \
        pk.PA_ERR_UNSUPPORTED
    assert lib.pa_decode_workspace_size(4, 66, 2, 128, 16, 100, ctypes.byref(nb), ctypes.byref(parts)) == \
        pk.PA_ERR_UNSUPPORTED  # group 33
    # groups above 8 run on the balanced schedule only
    assert lib.pa_decode_workspace_size_ex(4, 32, 2, 128, 16, 1000, 256, ctypes.byref(nb),
                                           ctypes.byref(parts), None) == pk.PA_ERR_UNSUPPORTED
    # ... and above 4096 requests on the tcgen05 consumer only, up to 32768
    assert lib.pa_decode_workspace_size_ex(5000, 32, 2, 128, 16, 1000, 0, ctypes.byref(nb),
                                           ctypes.byref(parts), None) == pk.PA_OK
    assert lib.pa_decode_workspace_size_ex(40000, 32, 2, 128, 16, 1000, 0, ctypes.byref(nb),
                                           ctypes.byref(parts), None) == pk.PA_ERR_UNSUPPORTED
    assert lib.pa_decode_workspace_size(4, 6, 4, 128, 16, 100, ctypes.byref(nb), ctypes.byref(parts)) == \
        pk.PA_ERR_INVALID
    # partition size must be a whole number of blocks
    assert lib.pa_decode_workspace_size_ex(4, 8, 2, 128, 16, 1000, 100, ctypes.byref(nb),
                                           ctypes.byref(parts), None) == pk.PA_ERR_INVALID
    # the balanced schedule on request only up to its batch limit; -2 is no schedule
    assert lib.pa_decode_workspace_size_ex(5000, 8, 2, 128, 16, 1000, -1, ctypes.byref(nb),
                                           ctypes.byref(parts), None) == pk.PA_ERR_UNSUPPORTED
    assert lib.pa_decode_workspace_size_ex(4, 8, 2, 128, 16, 1000, -2, ctypes.byref(nb),
                                           ctypes.byref(parts), None) == pk.PA_ERR_INVALID
    # batch 0 decode is a no-op
    assert lib.pa_decode(None, None, None, None, None, 0, 8, 2, 128, 16, 10, 4, 0, 1.0, None, 0, None) == pk.PA_OK
    assert lib.pa_selftest_wait_timeout(0, None) == pk.PA_ERR_INVALID


def test_explicit_partition_sizes_workspace():
    # explicit partitions do not consult the device
    nbytes, parts, sched = pk.pa_decode_workspace_size(2, 8, 2, 128, 16, 1000, partition_tokens=256,
                                                       with_schedule=True)
    assert parts == 4 and sched == "grid"
    rows = 2 * 8 * 4
    assert nbytes >= rows * 128 * 4 + 2 * rows * 4
    nbytes, parts = pk.pa_decode_workspace_size(2, 8, 2, 128, 16, 200, partition_tokens=256)
    assert (nbytes, parts) == (0, 1)


def test_allocator_errors():
    a = pk.PaAlloc(4, 2)
    a.add_seq(1)
    with pytest.raises(pk.PaError):
        a.add_seq(1)
    with pytest.raises(pk.PaError):
        a.free_seq(99)
    with pytest.raises(pk.PaError):
        a.fork(99, 3)
    with pytest.raises(pk.OutOfBlocks):
        a.append(1, 9)
    assert a.num_free() == 4 and a.seq_len(1) == 0
    with pytest.raises(pk.PaError):
        pk.PaAlloc(4, 2, initial_order=[0, 0, 1, 2])
