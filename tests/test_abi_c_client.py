"""A plain C99 program compiled against include/pa.h alone (gcc, no C++ or
CUDA headers) links libpa.so and drives the host-side calls: the worked
example of "Paged attention in LLMs" (section "A worked example": 14 tokens
in blocks of 5 fill 5/5/4 of 3 blocks, 15 slots held, 1 wasted), a fork and
its copy-on-write, an all-or-nothing append, and argument errors returned
before any launch.  No GPU needed."""

import json
import os
import shutil
import subprocess

import pytest

import paged_kv_cache_354_b200 as pk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden", "worked_example.json")


@pytest.fixture(scope="module")
def client_output(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path_factory.mktemp("abi") / "abi_client")
    libdir = os.path.dirname(pk.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "abi_client.c"), "-o", exe, "-L", libdir, "-lpa",
                    f"-Wl,-rpath,{libdir}"], check=True, capture_output=True, text=True)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0, res.stdout + res.stderr
    lines = {}
    for line in res.stdout.splitlines():
        key, *vals = line.split()
        lines[key] = vals
    assert "error" not in lines, lines.get("error")
    assert "done" in lines
    return lines


def test_worked_example_through_c(client_output):
    ex = json.load(open(GOLDEN))["worked_example"]["paged"]
    slots = [int(x) for x in client_output["slots"]]
    table = [int(x) for x in client_output["table"]]
    assert len(table) == ex["blocks"] == 3
    # every token's slot is block * 5 + offset, in order, through the table
    assert slots == [table[p // 5] * 5 + p % 5 for p in range(14)]
    fill = [sum(1 for s in slots if s // 5 == b) for b in table]
    assert fill == ex["fill"]
    tokens, logical, physical, live, free = (int(x) for x in client_output["stats"])
    assert (tokens, logical, physical, live, free) == (14, ex["held"], 3, 1, 8 - 3)
    assert logical - tokens == ex["wasted"]


def test_fork_and_copy_on_write_through_c(client_output):
    table = [int(x) for x in client_output["table"]]
    assert client_output["refcount_after_fork"] == ["2"]
    ncow, src, dst, _, slot = client_output["cow"]
    assert int(ncow) == 1 and int(src) == table[2] and int(dst) not in table
    # the child's table differs from the parent's only at the copied last block
    child = [int(x) for x in client_output["child_table"]]
    assert child[:2] == table[:2] and child[2] == int(dst)
    assert int(slot) == int(dst) * 5 + 4  # the 15th token: offset 4 of the copy


def test_errors_through_c(client_output):
    assert client_output["oom"][0] == "1" and client_output["oom"][2] == client_output["oom"][4]
    assert client_output["invalid"] == ["1", "msg"]
    assert client_output["empty_decode"] == ["1"]
    assert int(client_output["version"][0]) == pk.pa_version()
