"""Parity at the workloads' full sizes, in the launch configuration bench.py
times (auto variant, auto split-K partitions, one appended token per
request per step).

The GPU side runs exactly bench.py's state building and one decode step.
The oracle side replays the same seeded events on its own allocator model
and applies its own copy_blocks / reshape_and_cache to a host copy of the
pool taken before any of the library's kernels ran; it then computes
sampled (request, head) outputs one by one (full fp64 decode of every output
would take too long at these sizes).  Properties that hold at any size are
checked on every output.
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

SAMPLES = 24


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("name", ["tiny", "llama8b", "long", "beam", "mixed"])
def test_full_size_sampled(name):
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
    assert list(slots) == slots_r and len(pairs_r) == len(pairs)
    opa.copy_blocks(pool_u16, pairs_r)
    opa.reshape_and_cache(pool_u16, bits(ks[0]), bits(vs[0]), np.array(slots_r))
    t_ref, l_ref = workloads.block_tables(ref, ids_r)

    # properties on every output: finite, inside the range of the pool's values
    assert torch.isfinite(out).all()
    vmax = float(np.abs(u16_to_f64(np.array([(pool_u16[:, 1] & 0x7FFF).max()]))).max())
    assert out.float().abs().max().item() <= vmax + 1e-2

    # sampled outputs against the fp64 oracle (longest and shortest included)
    q64 = qs[0].double().cpu().numpy()
    got = out.double().cpu().numpy()
    rng = np.random.default_rng(workloads.seed_of(name) + 99)
    order = np.argsort(l_ref)
    reqs = [int(order[0]), int(order[-1])] + [int(x) for x in rng.integers(0, len(ids_r), SAMPLES - 2)]
    g = s.num_q_heads // s.num_kv_heads
    errs = []
    for b in reqs:
        n = int(l_ref[b])
        nblk = -(-n // s.block_size)
        j = int(rng.integers(0, s.num_q_heads))
        h = j // g
        # this request's blocks in table order, only its KV head (kept as a 1-head pool)
        mini = u16_to_f64(pool_u16[t_ref[b, :nblk]][:, :, h:h + 1])
        want = opa.decode_one(q64[b, j], mini, np.arange(nblk), n, 0, 1.0 / math.sqrt(s.head_dim))
        errs.append(np.abs(got[b, j] - want))
    errs = np.concatenate(errs)
    assert errs.max() <= MAX_ABS and errs.mean() <= MEAN_ABS, (errs.max(), errs.mean())


def test_full_size_multi_token_sampled():
    """pa_decode_multi at the Llama-3-8B decode shape with 4 causal query
    tokens per request (16 columns per KV head: the paired-warp kernel), the
    configuration of bench.py's multi-token study; sampled (request, token,
    head) outputs against the oracle over each token's visible prefix."""
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
    assert torch.isfinite(out).all()
    q64 = q.double().cpu().numpy()
    got = out.double().cpu().numpy()
    rng = np.random.default_rng(4242)
    g = s.num_q_heads // s.num_kv_heads
    errs = []
    for b in [int(x) for x in rng.integers(0, len(ids), SAMPLES)]:
        t = int(rng.integers(0, T))
        j = int(rng.integers(0, s.num_q_heads))
        h = j // g
        visible = int(lens[b]) - T + t + 1
        nblk = -(-visible // s.block_size)
        mini = u16_to_f64(pool_u16[tables[b, :nblk]][:, :, h:h + 1])
        want = opa.decode_one(q64[b, t, j], mini, np.arange(nblk), visible, 0, scale)
        errs.append(np.abs(got[b, t, j] - want))
    errs = np.concatenate(errs)
    assert errs.max() <= MAX_ABS and errs.mean() <= MEAN_ABS, (errs.max(), errs.mean())
