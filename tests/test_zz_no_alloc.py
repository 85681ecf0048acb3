"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: a plugin living inside a
host program that owns the GPU's whole memory budget and forbids its own
cudaMalloc calls, or a decode loop that cannot afford cudaMalloc's implicit
synchronisation.  pa_decode_noalloc keeps the split-K partials in a fixed
array compiled into the library instead.  These tests call it through the C
ABI and check it against pa_decode (caller workspace) on two calls in a row,
with inputs that need several sequence partitions, so the second call runs
over scratch the first one left behind.  Both entry points run the same plan
and kernels on the same inputs, so their outputs must be identical bit for
bit; each is also checked against the fp64 oracle.  The file is named to be
collected last; it passes alone in a fresh process as well.
"""

import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_354_b200 as pk
import workloads
from oracle import paged_attention as opa
from tests.gpu_helpers import bf16_to_f64, build_tables, compare, poison_unused, run_decode

pytestmark = pytest.mark.gpu

HQ, HKV, D, BS = 16, 4, 128, 16


def make_inputs(seed, lens):
    nb = sum(-(-int(n) // BS) for n in lens) + 8
    order = np.random.default_rng(seed).permutation(nb)
    t_ref, l_ref, tables, lens32, used = build_tables(lens, BS, nb, order)
    pool = poison_unused(workloads.bf16_normal((nb, 2, HKV, BS, D), seed=seed), used)
    q = workloads.bf16_normal((len(lens), HQ, D), seed=seed + 1)
    want = opa.decode(bf16_to_f64(q), bf16_to_f64(pool), t_ref, l_ref, 1.0 / np.sqrt(D))
    return q.cuda(), pool.cuda(), tables, lens32, want


def call_noalloc(q, pool, tables, lens, max_len, scale):
    out = torch.full_like(q, float("nan"))
    d_tables = torch.as_tensor(tables, device="cuda")
    d_lens = torch.as_tensor(lens, device="cuda")
    rc = pk.lib.pa_decode_noalloc(
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(pool.data_ptr()),
        ctypes.c_void_p(d_tables.data_ptr()), ctypes.c_void_p(d_lens.data_ptr()), q.shape[0], HQ, HKV, D, BS,
        pool.shape[0], tables.shape[1], int(max_len), float(scale),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == pk.PA_OK, pk.lib.pa_last_error_string().decode()
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("seeds", [(31, 32)])
def test_noalloc_matches_pa_decode_on_two_calls(seeds):
    cases = [
        (seeds[0], [3000, 17, 1200, 2049, 5, 640, 2999, 1]),
        (seeds[1], [1500, 2500, 33, 2047, 900, 16, 1024, 2900]),
    ]
    for seed, lens in cases:
        q, pool, tables, lens32, oracle_out = make_inputs(seed, lens)
        max_len = max(lens)
        nbytes, parts = pk.pa_decode_workspace_size(len(lens), HQ, HKV, D, BS, max_len)
        assert parts > 1, "the case must use split-K scratch"
        assert 0 < nbytes <= pk.PA_NOALLOC_SCRATCH_BYTES
        scale = 1.0 / np.sqrt(D)
        want = run_decode(q, pool, tables, lens32, scale)
        got = call_noalloc(q, pool, tables, lens32, max_len, scale)
        assert torch.isfinite(got).all()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), "differs from pa_decode"
        compare(bf16_to_f64(got), oracle_out)
        assert pk.pa_device_error() == 0


def test_noalloc_rejects_calls_beyond_its_scratch():
    # 8192 requests (above the balanced schedule's batch limit) x 64 heads x
    # 32768 tokens need far more scratch than the built-in array holds
    need, _ = pk.pa_decode_workspace_size(8192, 64, 8, 128, 16, 32768)
    assert need > pk.PA_NOALLOC_SCRATCH_BYTES
    rc = pk.lib.pa_decode_noalloc(None, None, None, None, None, 8192, 64, 8, 128, 16, 100000, 2048, 32768,
                                  0.1, None)
    assert rc == pk.PA_ERR_UNSUPPORTED
    assert "scratch" in pk.lib.pa_last_error_string().decode()
