"""pa_reshape_and_cache / pa_copy_blocks: bit-exact against the oracle.

The pool starts filled with a sentinel bit pattern so any stray write shows;
comparisons are on raw bf16 bits (as uint16).
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_354_b200 as pk
from oracle import paged_attention as opa
from oracle.block_allocator import BlockAllocator
import workloads

pytestmark = pytest.mark.gpu

SENTINEL = 0x7F81  # a signalling-NaN bit pattern no kernel writes


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("hkv,bs,d", [(2, 16, 128), (4, 16, 64), (8, 32, 128), (3, 5, 16)])
def test_reshape_and_cache_bit_exact(hkv, bs, d):
    nb, t = 13, 29
    rng = np.random.default_rng(hkv * 100 + bs)
    slots = rng.choice(nb * bs, size=t, replace=False).astype(np.int64)
    slots[[3, 11]] = -1  # padding tokens
    k = workloads.bf16_normal((t, hkv, d), seed=1)
    v = workloads.bf16_normal((t, hkv, d), seed=2)
    pool = torch.full((nb, 2, hkv, bs, d), SENTINEL, dtype=torch.int16).view(torch.bfloat16)
    want = opa.reshape_and_cache(bits(pool).copy(), bits(k), bits(v), slots)
    gpool = pool.cuda()
    pk.pa_reshape_and_cache(k.cuda(), v.cuda(), gpool, torch.as_tensor(slots, device="cuda"))
    torch.cuda.synchronize()
    assert np.array_equal(bits(gpool), want)
    assert pk.pa_device_error() == 0


def test_reshape_slot_out_of_pool_is_flagged():
    pool = torch.zeros((4, 2, 2, 16, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.ones((2, 2, 64), dtype=torch.bfloat16, device="cuda")
    pk.pa_device_error(clear=True)
    pk.pa_reshape_and_cache(k, k, pool, torch.tensor([3, 4 * 16], device="cuda"))
    torch.cuda.synchronize()
    assert pk.pa_device_error() == pk.PA_DEVERR_SLOT
    assert pool.float().sum().item() == 2 * 2 * 64  # only token 0 landed (K and V rows)


@pytest.mark.parametrize("hkv,bs,d", [(8, 16, 128), (2, 32, 64), (1, 16, 8)])
def test_copy_blocks_bit_exact(hkv, bs, d):
    nb = 40
    pool = workloads.bf16_normal((nb, 2, hkv, bs, d), seed=3)
    pairs = np.array([[1, 30], [5, 31], [5, 32], [17, 39], [0, 33]], dtype=np.int32)
    want = opa.copy_blocks(bits(pool).copy(), pairs)
    gpool = pool.cuda()
    pk.pa_copy_blocks(gpool, torch.as_tensor(pairs, device="cuda"))
    torch.cuda.synchronize()
    assert np.array_equal(bits(gpool), want)


def test_copy_pair_out_of_pool_is_flagged():
    pool = workloads.bf16_normal((6, 2, 2, 16, 64), seed=4).cuda()
    before = pool.clone()
    pk.pa_device_error(clear=True)
    pk.pa_copy_blocks(pool, torch.tensor([[0, 7], [-1, 2]], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert pk.pa_device_error() == pk.PA_DEVERR_COPY_PAIR
    assert torch.equal(pool, before)


def test_beam_copy_on_write_flow():
    """Prefix shared by 4 beams, 256 divergent tokens each: allocator pairs,
    copy_blocks then reshape_and_cache, bit-exact against the oracle flow.
    A smaller prefix than the full workload keeps the oracle fast."""
    hkv, bs, d = 2, 16, 64
    prompts, beams, prefix, grow = 3, 4, 2 * bs + 2, 40
    nb = 64
    order = np.random.default_rng(5).permutation(nb)
    ref, cpp = BlockAllocator(nb, bs, order), pk.PaAlloc(nb, bs, order)
    for a in (ref, cpp):
        for p in range(prompts):
            a.add_seq(100 + p)
            a.append(100 + p, prefix)
            for bm in range(beams):
                a.fork(100 + p, p * beams + bm)
            a.free_seq(100 + p)
    ids = list(range(prompts * beams))
    slots_r, pairs_r = ref.append_batch(ids, grow)
    slots_c, pairs_c = cpp.append_batch(ids, grow, as_numpy=True)
    assert len(pairs_r) == prompts * (beams - 1)
    pool = workloads.bf16_normal((nb, 2, hkv, bs, d), seed=6)
    k = workloads.bf16_normal((len(slots_r), hkv, d), seed=7)
    v = workloads.bf16_normal((len(slots_r), hkv, d), seed=8)
    want = opa.copy_blocks(bits(pool).copy(), pairs_r)
    want = opa.reshape_and_cache(want, bits(k), bits(v), np.array(slots_r))
    gpool = pool.cuda()
    pk.pa_copy_blocks(gpool, torch.as_tensor(pairs_c, device="cuda"))
    pk.pa_reshape_and_cache(k.cuda(), v.cuda(), gpool, torch.as_tensor(slots_c, device="cuda"))
    torch.cuda.synchronize()
    assert np.array_equal(bits(gpool), want)
