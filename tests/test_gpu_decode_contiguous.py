"""pa_decode_contiguous: decode over one reserved run per request (no block
table), against the fp64 oracle and against the paged decode.

Positions past each request's length in its reservation are NaN, so a
kernel that reads past the end fails.  Tolerance as for pa_decode: max
|err| <= 1e-2, mean |err| <= 1e-3.  On equal lengths the contiguous and the
paged decode run the same schedule and arithmetic, so their outputs must be
equal bit for bit -- checked at small sizes and at the Llama-3-8B shape.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_354_b200 as pk
import workloads
from oracle import paged_attention as opa
from tests.gpu_helpers import bf16_nan, bf16_to_f64, build_tables, compare, default_scale

pytestmark = pytest.mark.gpu

VARIANTS = {"auto": pk.PA_DECODE_AUTO, "cuda_core": pk.PA_DECODE_CUDA_CORE, "mma": pk.PA_DECODE_MMA}


def make_cache(lens, hkv, d, max_len, seed):
    cache = workloads.bf16_normal((len(lens), 2, hkv, max_len, d), seed=seed)
    for b, n in enumerate(lens):
        cache[b, :, :, int(n):] = bf16_nan()
    return cache


def run_contiguous(q, cache, lens, scale, variant="auto"):
    b, _, hkv, max_len, d = cache.shape
    ws = torch.empty(pk.pa_decode_contiguous_workspace_size(b, q.shape[1], hkv, d, max_len), dtype=torch.uint8,
                     device="cuda")
    out = torch.full_like(q, float("nan"))
    pk.pa_decode_contiguous(out, q, cache, torch.as_tensor(np.asarray(lens, dtype=np.int32), device="cuda"),
                            scale, ws, variant=VARIANTS[variant])
    torch.cuda.synchronize()
    return out


def paged_copy(cache, lens, bs, seed):
    """The same sequences in a shuffled paged pool (test-side marshalling)."""
    nb = sum(-(-int(n) // bs) for n in lens) + 3
    order = np.random.default_rng(seed).permutation(nb)
    _, _, tables, tlens, _ = build_tables(lens, bs, nb, order)
    _, _, hkv, _, d = cache.shape
    pool = torch.full((nb, 2, hkv, bs, d), float("nan"), dtype=torch.bfloat16)
    for b, n in enumerate(lens):
        for i in range(-(-int(n) // bs)):
            rows = min(bs, int(n) - i * bs)
            pool[int(tables[b, i]), :, :, :rows] = cache[b, :, :, i * bs:i * bs + rows]
    return pool, tables, tlens


RAGGED = [1, 15, 16, 17, 32, 53, 100, 257, 600, 0]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("variant,group", [("auto", 1), ("auto", 2), ("auto", 4), ("auto", 8),
                                           ("cuda_core", 4), ("mma", 1), ("mma", 3),
                                           ("auto", 16), ("mma", 12), ("mma", 24), ("auto", 32)])
def test_parity_with_oracle(d, variant, group):
    hkv, max_len = 2, 608
    cache = make_cache(RAGGED, hkv, d, max_len, seed=31 + group + d)
    q = workloads.bf16_normal((len(RAGGED), hkv * group, d), seed=32 + group)
    scale = default_scale(d)
    want = opa.decode_contiguous(bf16_to_f64(q), bf16_to_f64(cache), np.array(RAGGED), scale)
    out = run_contiguous(q.cuda(), cache.cuda(), RAGGED, scale, variant)
    assert pk.pa_device_error() == 0
    compare(bf16_to_f64(out), want)


@pytest.mark.parametrize("variant,group", [("auto", 4), ("cuda_core", 4), ("mma", 4), ("mma", 16), ("mma", 32)])
@pytest.mark.parametrize("lens", [RAGGED, [40000], [3, 0, 1]])
def test_bitwise_equal_to_paged(variant, group, lens):
    """Same lengths -> same units, same CTA ranges, same arithmetic (groups
    16 and 32: the grouped-warp mma.sync kernel in both layouts)."""
    hkv, d = 2, 128
    max_len = -(-max(lens) // 16) * 16 + 16
    cache = make_cache(lens, hkv, d, max_len, seed=41)
    q = workloads.bf16_normal((len(lens), hkv * group, d), seed=42)
    pool, tables, tlens = paged_copy(cache, lens, 16, seed=43)
    ws = torch.empty(1 << 24, dtype=torch.uint8, device="cuda")
    paged = torch.full_like(q, float("nan"), device="cuda")
    pk.pa_decode(paged, q.cuda(), pool.cuda(), torch.as_tensor(tables, device="cuda"),
                 torch.as_tensor(tlens, device="cuda"), max(lens), 0.09, workspace=ws, variant=VARIANTS[variant],
                 partition_tokens=pk.PA_SCHEDULE_BALANCED)
    contiguous = run_contiguous(q.cuda(), cache.cuda(), lens, 0.09, variant)
    assert pk.pa_device_error() == 0
    assert torch.equal(paged.view(torch.int16), contiguous.view(torch.int16))


def test_llama8b_shape_equal_to_paged_and_sampled_oracle():
    """The Llama-3-8B decode shape (B64, 32/8 heads, D128, lengths 512..4096)."""
    p = workloads.plan("llama8b")
    s = p.shape
    lens = [int(n) for n in p.seq_lens]
    max_len = -(-max(lens) // 16) * 16
    cache = make_cache(lens, s.num_kv_heads, s.head_dim, max_len, seed=51)
    q = workloads.bf16_normal((len(lens), s.num_q_heads, s.head_dim), seed=52)
    scale = default_scale(s.head_dim)
    out = run_contiguous(q.cuda(), cache.cuda(), lens, scale)
    pool, tables, tlens = paged_copy(cache, lens, 16, seed=53)
    ws = torch.empty(1 << 24, dtype=torch.uint8, device="cuda")
    paged = torch.empty_like(q, device="cuda")
    pk.pa_decode(paged, q.cuda(), pool.cuda(), torch.as_tensor(tables, device="cuda"),
                 torch.as_tensor(tlens, device="cuda"), max_len, scale, workspace=ws)
    torch.cuda.synchronize()
    assert pk.pa_device_error() == 0
    assert torch.equal(paged.view(torch.int16), out.view(torch.int16))
    rng = np.random.default_rng(54)
    for b in rng.choice(len(lens), size=6, replace=False):
        want = opa.decode_contiguous(bf16_to_f64(q[b:b + 1]), bf16_to_f64(cache[b:b + 1]), np.array([lens[b]]),
                                     scale)
        compare(bf16_to_f64(out[b:b + 1].cpu()), want)


def test_arguments_and_length_clamp():
    with pytest.raises(pk.PaError):
        pk.pa_decode_contiguous_workspace_size(4, 8, 2, 128, 100)  # max_len not a multiple of 16
    with pytest.raises(pk.PaError):
        pk.pa_decode_contiguous_workspace_size(5000, 8, 2, 128, 64)  # above the balanced batch limit
    lens = [20, 64]
    cache = make_cache(lens, 2, 128, 64, seed=61)
    q = workloads.bf16_normal((2, 8, 128), seed=62).cuda()
    pk.pa_device_error(clear=True)
    over = run_contiguous(q, cache.cuda(), [20, 70], 0.1)  # 70 > max_len: flagged, clamped to 64
    assert pk.pa_device_error() & pk.PA_DEVERR_SEQ_LEN
    exact = run_contiguous(q, cache.cuda(), lens, 0.1)
    assert pk.pa_device_error() == 0
    assert torch.equal(over.view(torch.int16), exact.view(torch.int16))
