"""bench.py's host-only paths keep their JSON contract (no GPU needed): the
reference arm (the fp64 oracle timed on the host) and the memory-waste study."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, timeout=600):
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                         timeout=timeout, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    return [json.loads(line) for line in res.stdout.splitlines() if line.startswith("{")]


def test_reference_arm_line():
    (line,) = run_bench("--impl", "reference", "--steps", "1", "--warmup", "3", "--cpu-seconds", "0.5",
                        "--workload", "tiny")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["steps"] == 1 and line["warmup"] == 3 and line["value"] > 0
    assert line["config"]["workload"].startswith("tiny: B4 Hq4/Hkv4 D64 bs16")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_memory_waste_study_lines():
    lines = run_bench("--study", "memory-waste")
    by_name = {ln["workload"]: ln for ln in lines}
    assert set(by_name) == {"tiny", "llama8b", "long", "beam", "mixed"}
    for ln in lines:
        # paged internal waste: under one block per request ("Paged attention in
        # LLMs": at most block_size - 1 slots in each request's last block)
        assert 0 <= ln["paged_logical_slots"] - ln["tokens"] <= ln["requests"] * (ln["block_size"] - 1)
        assert 0.0 <= ln["paged_internal_waste_frac"] < 1.0 and 0.0 <= ln["contiguous_waste_frac"] <= 1.0
    # varied lengths: reservation for the maximum wastes far more than paging
    for name in ("tiny", "llama8b", "mixed"):
        assert by_name[name]["contiguous_waste_frac"] > by_name[name]["paged_internal_waste_frac"]
    assert by_name["mixed"]["contiguous_waste_frac"] > 0.6 > 0.05 > by_name["mixed"]["paged_internal_waste_frac"]
    # beams sharing their prefix hold far fewer physical slots than tokens
    assert by_name["beam"]["paged_physical_over_tokens"] < 0.5


def test_committed_profiles_cite_one_capture():
    """The DRAM traffic that bench.py reports as roofline.traffic comes from
    profiles/paged_decode_traffic.json, and only while the decode sources hash
    to the digest stored there; every ncu summary under profiles/ names the
    sources it was captured on by that same digest, so the committed
    evidence is one capture of one set of sources."""
    import re

    with open(os.path.join(ROOT, "profiles", "paged_decode_traffic.json")) as f:
        rec = json.load(f)
    digests = {e["source_sha256"] for e in rec.values()}
    assert len(digests) == 1
    (digest,) = digests
    for e in rec.values():
        assert e["dram_read_bytes"] + e["dram_write_bytes"] == e["dram_bytes_per_launch"] > 0
    cited = {}
    for name in sorted(os.listdir(os.path.join(ROOT, "profiles"))):
        if name.endswith(".md"):
            with open(os.path.join(ROOT, "profiles", name)) as f:
                found = set(re.findall(r"`([0-9a-f]{64})`", f.read()))
            if found:
                cited[name] = found
    assert cited, "no summary names its sources"
    for name, found in cited.items():
        assert found == {digest}, name
