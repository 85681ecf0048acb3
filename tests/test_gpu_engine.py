"""The engine's serving step: C++ allocator into pinned staging, one H2D copy,
copy-on-write copies, and the cache write + decode + merge replayed from a
CUDA graph.  Every step is checked against the oracle's own replay of the
same events: allocator state, the pool bit for bit, and the decode output
within the attention tolerance.
"""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_354_b200 as pk
import workloads
from oracle import paged_attention as opa
from oracle.block_allocator import BlockAllocator
from paged_kv_cache_354_b200.engine import PagedDecodeCache
from tests.gpu_helpers import compare, u16_to_f64

pytestmark = pytest.mark.gpu


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("schedule", [0, 256])
def test_graph_replayed_steps_match_oracle(schedule):
    dev = torch.device("cuda", torch.cuda.current_device())
    hq, hkv, d, bs = 32, 8, 128, 16
    nb = 600
    order = np.random.default_rng(7).permutation(nb)
    cache = PagedDecodeCache(nb, hq, hkv, d, bs, max_batch=6, max_seq_len=2200, initial_order=order,
                             device=dev, partition_tokens=schedule)
    ref = BlockAllocator(nb, bs, order)
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    cache.pool.copy_(torch.randn(cache.pool.shape, generator=gen, device=dev).bfloat16())
    pool_ref = bits(cache.pool)
    # two prompts, each forked into beams sharing a partial last block
    for a in (cache.alloc, ref):
        a.add_seq(100)
        a.append(100, 1000 + 7)
        a.add_seq(101)
        a.append(101, 2000 + 3)
        for beam in range(3):
            a.fork(100, beam)
        for beam in range(3, 6):
            a.fork(101, beam)
        a.free_seq(100)
        a.free_seq(101)
    ids = list(range(6))
    out = torch.empty((6, hq, d), dtype=torch.bfloat16, device=dev)
    scale = 1.0 / math.sqrt(d)

    def oracle_step(qh, kh, vh):
        slots, pairs = ref.append_batch(ids, 1)
        opa.copy_blocks(pool_ref, pairs)
        opa.reshape_and_cache(pool_ref, bits(kh), bits(vh), np.array(slots))
        tables, lens = workloads.block_tables(ref, ids, cache.max_blocks)
        want = opa.decode(qh.double().numpy(), u16_to_f64(pool_ref), tables, lens, scale)
        return slots, pairs, tables, lens, want

    seen_cow = 0
    for step in range(4):
        qh = torch.randn((6, hq, d), generator=torch.Generator().manual_seed(step)).bfloat16()
        kh = torch.randn((6, hkv, d), generator=torch.Generator().manual_seed(100 + step)).bfloat16()
        vh = torch.randn((6, hkv, d), generator=torch.Generator().manual_seed(200 + step)).bfloat16()
        npairs = cache.host_step(ids)
        slots, pairs, tables, lens, want = oracle_step(qh, kh, vh)
        # the allocator's staged output equals the oracle's
        assert cache.staged("slots").numpy().tolist() == list(slots)
        assert npairs == len(pairs)
        assert [tuple(p) for p in cache.staged("pairs")[:npairs].numpy().tolist()] == [tuple(p) for p in pairs]
        assert np.array_equal(cache.staged("tables").numpy(), tables)
        assert np.array_equal(cache.staged("lens").numpy(), lens)
        seen_cow += npairs
        cache.staged("q").copy_(qh)
        cache.staged("k").copy_(kh)
        cache.staged("v").copy_(vh)
        cache.upload()
        if step == 0:
            # record the device part on this step's staged data; the capture's
            # warm-up already performs this step's copies and cache write
            if npairs:
                pk.pa_copy_blocks(cache.pool, cache.s_pairs[:npairs])
            cache.capture(out)
        else:
            cache.replay(npairs)
        torch.cuda.synchronize()
        assert np.array_equal(bits(cache.pool), pool_ref), f"pool differs after step {step}"
        compare(out.double().cpu().numpy(), want)
    assert seen_cow == 4  # 2 + 2 beams copy their prompt's shared partial block on step 0
    assert pk.pa_device_error() == 0


@pytest.mark.parametrize("zero_copy,hq", [(True, 8), (False, 8), (True, 32), (True, 48)])
def test_whole_step_graphs_match_oracle(zero_copy, hq):
    """capture_steps: upload and fused decode as one graph per staging
    buffer, the output reaching pinned host memory straight from the kernels
    (zero_copy) or through a device-to-host copy in the graph (steps with
    copy-on-write pairs -- here step 3 -- run eagerly); every step's host
    output equals the oracle's replay, and the pool equals the oracle's bit
    for bit."""
    dev = torch.device("cuda", torch.cuda.current_device())
    hkv, d, bs, sets = 2, 128, 16, 3  # hq 32 / 48: groups 16 / 24 on the tcgen05 consumer
    nb = 200
    order = np.random.default_rng(11).permutation(nb)
    cache = PagedDecodeCache(nb, hq, hkv, d, bs, max_batch=4, max_seq_len=700, initial_order=order,
                             device=dev, staging_sets=sets)
    ref = BlockAllocator(nb, bs, order)
    gen = torch.Generator(device=dev)
    gen.manual_seed(12)
    cache.pool.copy_(torch.randn(cache.pool.shape, generator=gen, device=dev).bfloat16())
    pool_ref = bits(cache.pool)
    for a in (cache.alloc, ref):
        a.add_seq(0)
        a.append(0, 300 + 5)
        a.fork(0, 1)  # shares a partial block: the first step copies it
        for sid, n in ((2, 17), (3, 640)):
            a.add_seq(sid)
            a.append(sid, n)
    ids = [0, 1, 2, 3]
    out = torch.empty((4, hq, d), dtype=torch.bfloat16, device=dev)
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    scale = 1.0 / math.sqrt(d)
    inputs = []
    for step in range(7):
        g = torch.Generator().manual_seed(50 + step)
        inputs.append(tuple(torch.randn(shape, generator=g).bfloat16()
                            for shape in ((4, hq, d), (4, hkv, d), (4, hkv, d))))
    for j in range(sets):  # the first steps' inputs, as the loop below stages them
        for name, t in zip("qkv", inputs[j]):
            cache.staged(name, j).copy_(t)
    npairs = cache.host_step(ids, 0)
    assert npairs == 1
    cache.upload(0)
    pk.pa_copy_blocks(cache.pool, cache.s_pairs[:npairs])
    cache.capture(out)  # its warm-up performs step 0
    cache.capture_steps(out, h_out, zero_copy=zero_copy)
    torch.cuda.synchronize()
    seen = 0
    for step in range(7):
        j = step % sets
        if step == 3:  # request 2 restarts as a fork of request 3: its first write copies
            for a in (cache.alloc, ref):
                a.free_seq(2)
                a.fork(3, 2)
        if step > 0:
            for name, t in zip("qkv", inputs[step]):
                cache.staged(name, j).copy_(t)
            npairs = cache.host_step(ids, j)
            assert npairs == (1 if step == 3 else 0)
            cache.replay_step(j, npairs)
        else:
            h_out.copy_(out)
        torch.cuda.synchronize()
        slots, pairs = ref.append_batch(ids, 1)
        assert len(pairs) == npairs
        seen += npairs
        opa.copy_blocks(pool_ref, pairs)
        qh, kh, vh = inputs[step]
        opa.reshape_and_cache(pool_ref, bits(kh), bits(vh), np.array(slots))
        tables, lens = workloads.block_tables(ref, ids, cache.max_blocks)
        want = opa.decode(qh.double().numpy(), u16_to_f64(pool_ref), tables, lens, scale)
        compare(h_out.double().numpy(), want)
    assert seen == 2
    assert np.array_equal(bits(cache.pool), pool_ref)
    assert pk.pa_device_error() == 0
