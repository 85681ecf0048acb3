"""Parity at the workloads' full sizes, in the launch configuration bench.py
times (auto variant, auto split-K partitions, one appended token per
request per step).

The GPU side runs exactly bench.py's state building and one decode step.
The oracle side replays the same seeded events on its own allocator model
and applies its own copy_blocks / reshape_and_cache to a host copy of the
pool taken before any of the library's kernels ran.  Then:

* the whole pool after the step must equal the oracle's pool bit for bit
  (copy-on-write copies, the fused cache write, and nothing else touched);
* every (request, query head) output is compared with the fp64 oracle's
  decode of that request, max |err| <= 1e-2 and mean |err| <= 1e-3.

The oracle decodes one request at a time over a small pool holding only
that request's blocks (in table order), so the full pool never needs an
fp64 copy; at these sizes the whole batch takes seconds on one host core.
"""

import math

import numpy as np
import pytest
import torch

import bench
import paged_kv_cache_354_b200 as pk
import workloads
from oracle import paged_attention as opa
from oracle.block_allocator import BlockAllocator
from tests.gpu_helpers import MAX_ABS, MEAN_ABS, u16_to_f64

pytestmark = pytest.mark.gpu


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_batch(q64, pool_u16, tables, lens, bs, scale):
    """fp64 oracle output of every (request, query head): [B, Hq, D]."""
    out = np.zeros(q64.shape, dtype=np.float64)
    for b in range(q64.shape[0]):
        n = int(lens[b])
        nblk = -(-n // bs)
        mini = u16_to_f64(pool_u16[tables[b, :nblk]])
        out[b] = opa.decode(q64[b:b + 1], mini, np.arange(nblk)[None, :], np.array([n]), scale)[0]
    return out


def oracle_batch_multi(q64, pool_u16, tables, lens, bs, scale):
    """fp64 oracle of every (request, query token, query head) of a causal
    multi-token decode, q64 [B, T, Hq, D]; one request and KV head at a time
    (a one-head pool of that request's blocks)."""
    batch, _, hq, _ = q64.shape
    hkv = pool_u16.shape[2]
    g = hq // hkv
    out = np.zeros(q64.shape, dtype=np.float64)
    for b in range(batch):
        n = int(lens[b])
        nblk = -(-n // bs)
        blocks = pool_u16[tables[b, :nblk]]
        for h in range(hkv):
            mini = u16_to_f64(blocks[:, :, h:h + 1])
            out[b, :, h * g:(h + 1) * g] = opa.decode_multi(q64[b:b + 1, :, h * g:(h + 1) * g], mini,
                                                            np.arange(nblk)[None, :], np.array([n]), scale)[0]
    return out


def assert_close(got, want):
    err = np.abs(got - want)
    assert np.isfinite(got).all(), "non-finite output"
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    return err


@pytest.mark.parametrize("name", ["tiny", "llama8b", "long", "beam", "mixed"])
def test_full_size_whole_batch(name):
    dev = torch.device("cuda", torch.cuda.current_device())
    p, cache, ids, gen = bench.build_cache(name, 2, 0, dev, prefill=False)
    s = p.shape
    pool_u16 = bits(cache.pool)  # host snapshot before any library kernel
    ref = BlockAllocator(p.num_blocks, s.block_size, p.initial_order)
    ids_r = workloads.populate(ref, p)
    assert ids_r == ids
    pk.pa_device_error(clear=True)

    if name == "beam":
        slots, pairs, k, v = bench.beam_prefill(p, cache, ids, gen, dev)
        slots_r, pairs_r = ref.append_batch(ids_r, p.append_tokens)
        assert len(pairs_r) == 24
        assert list(slots) == slots_r and [tuple(x) for x in pairs] == pairs_r
        opa.copy_blocks(pool_u16, pairs_r)
        opa.reshape_and_cache(pool_u16, bits(k), bits(v), np.array(slots_r))

    # one step exactly as bench.py runs it
    qs, ks, vs = bench.make_inputs(cache, len(ids), gen, dev)
    slots, pairs, tables, lens = cache.plan_append(ids)
    out = torch.full_like(qs[0], float("nan"))
    cache.run(qs[0], ks[0], vs[0], out, torch.as_tensor(slots, device=dev), torch.as_tensor(tables, device=dev),
              torch.as_tensor(lens, device=dev), torch.as_tensor(pairs.reshape(-1, 2), device=dev))
    torch.cuda.synchronize()
    assert pk.pa_device_error() == 0

    slots_r, pairs_r = ref.append_batch(ids_r, 1)
    assert list(slots) == slots_r and [tuple(x) for x in pairs] == pairs_r
    opa.copy_blocks(pool_u16, pairs_r)
    opa.reshape_and_cache(pool_u16, bits(ks[0]), bits(vs[0]), np.array(slots_r))
    t_ref, l_ref = workloads.block_tables(ref, ids_r)
    assert np.array_equal(lens, l_ref)

    # the whole pool, bit for bit: copy-on-write copies and the cache write
    assert np.array_equal(bits(cache.pool), pool_u16), "pool differs from the oracle's"

    # every output against the fp64 oracle
    want = oracle_batch(qs[0].double().cpu().numpy(), pool_u16, t_ref, l_ref, s.block_size,
                        1.0 / math.sqrt(s.head_dim))
    assert_close(out.double().cpu().numpy(), want)


def test_full_size_multi_token_whole_batch():
    """pa_decode_multi at the Llama-3-8B decode shape with 4 causal query
    tokens per request (16 columns per KV head), the configuration of
    bench.py's multi-token study: every (request, token, head) output
    against the oracle over that token's visible prefix."""
    dev = torch.device("cuda", torch.cuda.current_device())
    p, cache, ids, gen = bench.build_cache("llama8b", 2, 0, dev, prefill=False)
    s = p.shape
    T = 4
    pool_u16 = bits(cache.pool)
    tables, lens = cache.alloc.block_tables(ids, cache.max_blocks)
    q = torch.randn((len(ids), T, s.num_q_heads, s.head_dim), generator=gen, device=dev).bfloat16()
    out = torch.full_like(q, float("nan"))
    scale = 1.0 / math.sqrt(s.head_dim)
    ws = torch.empty(max(256, pk.pa_decode_multi_workspace_size(len(ids), T, s.num_q_heads, s.num_kv_heads,
                                                                 s.head_dim, s.block_size, cache.max_seq_len)),
                     dtype=torch.uint8, device=dev)
    pk.pa_device_error(clear=True)
    pk.pa_decode_multi(out, q, cache.pool, torch.as_tensor(tables, device=dev), torch.as_tensor(lens, device=dev),
                       cache.max_seq_len, scale, ws)
    torch.cuda.synchronize()
    assert pk.pa_device_error() == 0
    ref = BlockAllocator(p.num_blocks, s.block_size, p.initial_order)
    ids_r = workloads.populate(ref, p)
    t_ref, l_ref = workloads.block_tables(ref, ids_r)
    want = oracle_batch_multi(q.double().cpu().numpy(), pool_u16, t_ref, l_ref, s.block_size, scale)
    assert_close(out.double().cpu().numpy(), want)


@pytest.mark.parametrize("group", [16, 32])
def test_full_size_wide_group_whole_batch(group):
    """The Llama-3-8B decode workload's lengths, pool and tables with 16 or 32
    query heads per KV head (the tcgen05 consumer): every output against the
    oracle."""
    dev = torch.device("cuda", torch.cuda.current_device())
    p, cache, ids, gen = bench.build_cache("llama8b", 2, 0, dev, prefill=False)
    s = p.shape
    hq = s.num_kv_heads * group
    pool_u16 = bits(cache.pool)
    tables, lens = cache.alloc.block_tables(ids, cache.max_blocks)
    q = torch.randn((len(ids), hq, s.head_dim), generator=gen, device=dev).bfloat16()
    out = torch.full_like(q, float("nan"))
    scale = 1.0 / math.sqrt(s.head_dim)
    nbytes, _ = pk.pa_decode_workspace_size(len(ids), hq, s.num_kv_heads, s.head_dim, s.block_size,
                                            cache.max_seq_len)
    ws = torch.empty(max(256, nbytes), dtype=torch.uint8, device=dev)
    pk.pa_device_error(clear=True)
    pk.pa_decode(out, q, cache.pool, torch.as_tensor(tables, device=dev), torch.as_tensor(lens, device=dev),
                 cache.max_seq_len, scale, workspace=ws)
    torch.cuda.synchronize()
    assert pk.pa_device_error() == 0
    ref = BlockAllocator(p.num_blocks, s.block_size, p.initial_order)
    t_ref, l_ref = workloads.block_tables(ref, workloads.populate(ref, p))
    want = oracle_batch(q.double().cpu().numpy(), pool_u16, t_ref, l_ref, s.block_size, scale)
    assert_close(out.double().cpu().numpy(), want)
