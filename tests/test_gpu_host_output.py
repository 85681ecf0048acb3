"""Decode output stored straight into pinned host memory (zero-copy).

The decode calls accept an ``out`` in page-locked host memory that the
device addresses at the same pointer; the kernels then store every output
row across PCIe.  The arithmetic does not change, so each case must give
the same bits as the same call with ``out`` on the device, and every row
must be written (the host buffer starts as NaN).  Pageable host memory is
refused before any launch.
"""

import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_354_b200 as pk
import workloads
from oracle import paged_attention as opa
from tests.gpu_helpers import bf16_to_f64, build_tables, compare, poison_unused, workspace_for

pytestmark = pytest.mark.gpu

LENS = [1, 17, 250, 3000, 0, 1024, 2049, 33, 640, 4096, 5, 1500]


def make(lens, hq, hkv, d, bs, seed, T=None):
    nb = sum(-(-int(n) // bs) for n in lens) + 4
    order = np.random.default_rng(seed).permutation(nb)
    t_ref, l_ref, t_cpp, l_cpp, used = build_tables(lens, bs, nb, order)
    pool = poison_unused(workloads.bf16_normal((nb, 2, hkv, bs, d), seed=seed), used)
    shape = (len(lens), hq, d) if T is None else (len(lens), T, hq, d)
    q = workloads.bf16_normal(shape, seed=seed + 1)
    dev = torch.device("cuda")
    return (q.to(dev), pool.to(dev), torch.as_tensor(t_cpp, device=dev), torch.as_tensor(l_cpp, device=dev),
            (q, pool, t_ref, l_ref))


def pinned_nan(like):
    return torch.full(like.shape, float("nan"), dtype=like.dtype).pin_memory()


def both(call, like):
    """call(out) with out on the device, then with out in pinned host memory."""
    d_out = torch.full_like(like, float("nan"))
    call(d_out)
    h_out = pinned_nan(like)
    call(h_out)
    torch.cuda.synchronize()
    assert pk.pa_device_error() == 0
    return d_out.cpu(), h_out


# (variant, schedule, hq, hkv, d, bs): mma.sync on the balanced schedule and
# on the per-partition grid (split-K merge writes too), the block-pair tile,
# the CUDA-core consumer, a wide group on paired warps, the tcgen05 consumer
CASES = [
    (pk.PA_DECODE_AUTO, 0, 32, 8, 128, 16),
    (pk.PA_DECODE_MMA, 64, 8, 2, 128, 16),
    (pk.PA_DECODE_AUTO, 0, 8, 2, 64, 16),
    (pk.PA_DECODE_CUDA_CORE, pk.PA_SCHEDULE_BALANCED, 4, 2, 128, 32),
    (pk.PA_DECODE_MMA, pk.PA_SCHEDULE_BALANCED, 64, 2, 128, 16),
    (pk.PA_DECODE_TCGEN05, pk.PA_SCHEDULE_BALANCED, 32, 2, 128, 16),
]


@pytest.mark.parametrize("variant,schedule,hq,hkv,d,bs", CASES)
def test_decode_into_pinned_host_memory(variant, schedule, hq, hkv, d, bs):
    q, pool, tables, lens, (qh, poolh, t_ref, l_ref) = make(LENS, hq, hkv, d, bs, seed=700 + hq + d + bs)
    max_len = max(LENS)
    ws_sched = pk.PA_SCHEDULE_BALANCED if variant == pk.PA_DECODE_TCGEN05 else schedule
    ws, _ = workspace_for(len(LENS), hq, hkv, d, bs, max_len, ws_sched)
    scale = 0.09
    dev, host = both(lambda out: pk.pa_decode(out, q, pool, tables, lens, max_len, scale, workspace=ws,
                                              variant=variant, partition_tokens=schedule), q)
    assert torch.equal(host.view(torch.int16), dev.view(torch.int16))
    compare(bf16_to_f64(host), opa.decode(bf16_to_f64(qh), bf16_to_f64(poolh), t_ref, l_ref, scale))


def test_decode_append_into_pinned_host_memory():
    """The fused cache write + decode: same output bits and the same pool."""
    lens = [40, 300, 16, 1000, 7, 2500]
    hq, hkv, d, bs = 32, 8, 128, 16
    q, pool, tables, lens_d, _ = make(lens, hq, hkv, d, bs, seed=731)
    # each request's newest token sits at position len - 1: rewrite it
    slots = []
    for b, n in enumerate(lens):
        blk = int(tables[b, (n - 1) // bs])
        slots.append(blk * bs + (n - 1) % bs)
    slots = torch.as_tensor(slots, dtype=torch.int64, device="cuda")
    k = workloads.bf16_normal((len(lens), hkv, d), seed=732).cuda()
    v = workloads.bf16_normal((len(lens), hkv, d), seed=733).cuda()
    ws, _ = workspace_for(len(lens), hq, hkv, d, bs, max(lens))
    pool2 = pool.clone()
    d_out = torch.full_like(q, float("nan"))
    pk.pa_decode_append(d_out, q, pool, k, v, slots, tables, lens_d, max(lens), 0.088, workspace=ws)
    h_out = pinned_nan(q)
    pk.pa_decode_append(h_out, q, pool2, k, v, slots, tables, lens_d, max(lens), 0.088, workspace=ws)
    torch.cuda.synchronize()
    assert pk.pa_device_error() == 0
    assert torch.equal(h_out.view(torch.int16), d_out.cpu().view(torch.int16))
    assert torch.equal(pool2.view(torch.int16), pool.view(torch.int16))


@pytest.mark.parametrize("T,hq,hkv", [(2, 8, 2), (4, 8, 2), (3, 32, 4)])
def test_decode_multi_into_pinned_host_memory(T, hq, hkv):
    lens = [T, 50, 700, 2049, 1]
    q, pool, tables, lens_d, _ = make(lens, hq, hkv, 128, 16, seed=740 + T, T=T)
    ws = torch.empty(max(256, pk.pa_decode_multi_workspace_size(len(lens), T, hq, hkv, 128, 16, max(lens))),
                     dtype=torch.uint8, device="cuda")
    dev, host = both(lambda out: pk.pa_decode_multi(out, q, pool, tables, lens_d, max(lens), 0.088, ws), q)
    assert torch.equal(host.view(torch.int16), dev.view(torch.int16))


def test_decode_contiguous_into_pinned_host_memory():
    lens = [1, 64, 333, 1024]
    hq, hkv, d, max_len = 16, 4, 128, 1024
    cache = workloads.bf16_normal((len(lens), 2, hkv, max_len, d), seed=750).cuda()
    q = workloads.bf16_normal((len(lens), hq, d), seed=751).cuda()
    lens_d = torch.as_tensor(lens, dtype=torch.int32, device="cuda")
    ws = torch.empty(pk.pa_decode_contiguous_workspace_size(len(lens), hq, hkv, d, max_len), dtype=torch.uint8,
                     device="cuda")
    dev, host = both(lambda out: pk.pa_decode_contiguous(out, q, cache, lens_d, 0.088, ws), q)
    assert torch.equal(host.view(torch.int16), dev.view(torch.int16))


def test_pageable_host_output_is_refused():
    """Through the C ABI directly (the binding refuses it earlier): an out
    pointer into pageable host memory returns PA_ERR_INVALID and launches
    nothing; the binding raises TypeError for a CPU tensor that is not pinned."""
    q, pool, tables, lens, _ = make([100, 200], 8, 2, 128, 16, seed=760)
    ws, _ = workspace_for(2, 8, 2, 128, 16, 200)
    pageable = np.full(q.numel(), 0x7FC0, dtype=np.uint16)  # bf16 NaN bits
    pk.pa_device_error(clear=True)
    rc = pk.lib.pa_decode_ex(ctypes.c_void_p(pageable.ctypes.data), pk._ptr(q), pk._ptr(pool), pk._ptr(tables),
                             pk._ptr(lens), 2, 8, 2, 128, 16, pool.shape[0], tables.shape[1], 200,
                             ctypes.c_float(0.088), pk._ptr(ws), ws.numel(), pk.PA_DECODE_AUTO, 0,
                             pk._stream(None))
    torch.cuda.synchronize()
    assert rc == pk.PA_ERR_INVALID
    assert (pageable == 0x7FC0).all()
    assert pk.pa_device_error() == 0
    with pytest.raises(TypeError):
        pk.pa_decode(torch.empty(q.shape, dtype=torch.bfloat16), q, pool, tables, lens, 200, 0.088, workspace=ws)
