"""pa_decode_append (cache write of each request's newest token fused with
decode) gives exactly what pa_reshape_and_cache followed by pa_decode gives:
the same output bits and the same pool bits, on both schedules, with padding
slots and empty requests; and it matches the oracle."""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_354_b200 as pk
import workloads
from oracle import paged_attention as opa
from oracle.block_allocator import BlockAllocator
from tests.gpu_helpers import compare, u16_to_f64, workspace_for

pytestmark = pytest.mark.gpu


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("lens,hq,hkv,d,bs", [
    ([700, 1, 2049, 64, 300, 1500, 17, 1024], 32, 8, 128, 16),   # balanced schedule
    ([900, 33, 5, 2047, 400], 16, 4, 64, 32),                      # balanced, other shape
    ([3, 20, 1], 4, 4, 64, 16),                                    # little work: per-partition grid
    ([900, 33, 5, 2047, 400, 1600, 2500, 3000], 16, 4, 64, 16),   # balanced on block pairs: stored before the TMA load
    ([700, 1, 2049, 64, 300, 1500, 17, 1024], 32, 2, 128, 16),    # group 16 (tcgen05): stored before the TMA load
    ([700, 1, 2049, 64, 300, 1500, 17, 1024], 48, 2, 128, 32),    # group 24 (tcgen05, two halves), bs32
    ([900, 33, 5, 2047, 400, 128, 127, 129], 64, 4, 128, 16),     # group 16, tile edges
    ([700, 1, 2049, 64, 300, 1500, 17, 1024], 32, 2, 64, 16),     # group 16 at head dim 64 (paired warps, pairs)
    ([700, 1, 2049, 64, 300, 1500, 17, 1024], 64, 2, 64, 32),     # group 32 at head dim 64 (four warps per block)
    ([int(x) for x in np.random.default_rng(67).integers(1, 30, size=4200)], 32, 2, 64, 16),  # 4200 requests: tcgen05
    # 512 / 513 requests: the merge kernel (which stores the new rows on this
    # path) computes the prefix sums itself, or reads the decode kernel's copy
    ([int(x) for x in np.random.default_rng(68).integers(1, 200, size=512)], 8, 2, 128, 16),
    ([int(x) for x in np.random.default_rng(69).integers(1, 200, size=513)], 8, 2, 128, 16),
])
def test_append_equals_separate_calls(lens, hq, hkv, d, bs):
    dev = torch.device("cuda", torch.cuda.current_device())
    nb = sum(-(-(n + 1) // bs) for n in lens) + 8
    order = np.random.default_rng(len(lens)).permutation(nb)
    cpp, ref = pk.PaAlloc(nb, bs, order), BlockAllocator(nb, bs, order)
    ids = list(range(len(lens)))
    for a in (cpp, ref):
        for sid, n in zip(ids, lens):
            a.add_seq(sid)
            a.append(sid, n)
    slots, _ = cpp.append_batch(ids, 1, as_numpy=True)
    slots_r, _ = ref.append_batch(ids, 1)
    assert list(slots) == slots_r
    slots[1] = -1  # one padding token: nothing written, decode reads the pool's row
    slots_r[1] = -1
    mb = max(-(-(n + 1) // bs) for n in lens)
    tables, lens1 = cpp.block_tables(ids, mb)
    pool = workloads.bf16_normal((nb, 2, hkv, bs, d), seed=3).to(dev)
    q = workloads.bf16_normal((len(lens), hq, d), seed=4).to(dev)
    k = workloads.bf16_normal((len(lens), hkv, d), seed=5).to(dev)
    v = workloads.bf16_normal((len(lens), hkv, d), seed=6).to(dev)
    d_slots = torch.as_tensor(slots, device=dev)
    d_t, d_l = torch.as_tensor(tables, device=dev), torch.as_tensor(lens1, device=dev)
    max_len = int(lens1.max())
    scale = 1.0 / math.sqrt(d)
    pool_start = bits(pool)
    # separate calls
    pool_a = pool.clone()
    out_a = torch.empty_like(q)
    ws, _ = workspace_for(len(lens), hq, hkv, d, bs, max_len)
    pk.pa_reshape_and_cache(k, v, pool_a, d_slots)
    pk.pa_decode(out_a, q, pool_a, d_t, d_l, max_len, scale, workspace=ws)
    # fused
    pool_b = pool.clone()
    out_b = torch.empty_like(q)
    pk.pa_decode_append(out_b, q, pool_b, k, v, d_slots, d_t, d_l, max_len, scale, workspace=ws)
    torch.cuda.synchronize()
    assert pk.pa_device_error() == 0
    assert torch.equal(out_a, out_b)
    assert np.array_equal(bits(pool_a), bits(pool_b))
    # and the oracle
    want_pool = opa.reshape_and_cache(pool_start.copy(), bits(k), bits(v), np.array(slots_r))
    assert np.array_equal(bits(pool_b), want_pool)
    t_ref, l_ref = workloads.block_tables(ref, ids, mb)
    want = opa.decode(q.double().cpu().numpy(), u16_to_f64(want_pool), t_ref, l_ref, scale)
    if len(lens) <= 64:
        compare(out_b.double().cpu().numpy(), want)
    else:
        # hundreds of requests, some of a few positions: the bf16 probabilities
        # and output can move an element by 2^-8 (|v - out| spread + |out|)
        # beyond 1e-2 (tests/test_gpu_decode.py, check_short); |v| < ~5.5 here
        err = np.abs(out_b.double().cpu().numpy() - want)
        assert err.mean() <= 1e-3 and (err <= 1e-2 + 2.0 ** -8 * (11.0 + np.abs(want))).all()


@pytest.mark.parametrize("hq,d", [(8, 128), (32, 128), (32, 64)])
def test_append_with_empty_requests(hq, d):
    """Empty requests with and without a slot (one writes into a block no
    request holds: only the cache write touches it); group 4 on mma.sync,
    group 16 on the tcgen05 consumer, group 16 at head dim 64 on paired
    warps over block pairs."""
    dev = torch.device("cuda", torch.cuda.current_device())
    hkv, bs = 2, 16
    lens = [0, 1500, 0, 2000] * 8  # 32 requests, enough work for the balanced schedule
    nb = sum(-(-n // bs) for n in lens) + 4
    a = pk.PaAlloc(nb, bs)
    ids = list(range(len(lens)))
    for sid, n in zip(ids, lens):
        a.add_seq(sid)
        if n:
            a.append(sid, n - 1)
    live = [sid for sid, n in zip(ids, lens) if n]
    slots_live, _ = a.append_batch(live, 1, as_numpy=True)
    slots = np.full(len(lens), -1, dtype=np.int64)
    slots[live] = slots_live
    slots[2] = (nb - 1) * bs + 3  # an empty request with a slot, in the last (free) block
    tables, l = a.block_tables(ids, max(-(-n // bs) for n in lens))
    assert list(l) == lens
    pool = workloads.bf16_normal((nb, 2, hkv, bs, d), seed=7).to(dev)
    q = workloads.bf16_normal((len(lens), hq, d), seed=8).to(dev)
    k = workloads.bf16_normal((len(lens), hkv, d), seed=9).to(dev)
    v = workloads.bf16_normal((len(lens), hkv, d), seed=10).to(dev)
    ws, _ = workspace_for(len(lens), hq, hkv, d, bs, 2000)
    out = torch.full_like(q, float("nan"))
    d_slots, d_t, d_l = (torch.as_tensor(x, device=dev) for x in (slots, tables, l))
    before = pool.clone()
    pk.pa_decode_append(out, q, pool, k, v, d_slots, d_t, d_l, 2000, 0.1, workspace=ws)
    ref_pool = before.clone()
    pk.pa_reshape_and_cache(k, v, ref_pool, d_slots)
    ref_out = torch.empty_like(q)
    pk.pa_decode(ref_out, q, ref_pool, d_t, d_l, 2000, 0.1, workspace=ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out[0]) == 0 and torch.equal(out, ref_out)
    assert torch.equal(pool, ref_pool)
