"""pa_decode parity with the fp64 oracle on small and ragged cases.

Sizes span several partitions, stages and tiles with a ragged tail; every
pool row that holds no token is NaN, so a kernel that reads past a request's
end, or lets P=0 meet a NaN value, fails.  Tolerance (attention outputs vs
fp64): max |err| <= 1e-2 and mean |err| <= 1e-3.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_354_b200 as pk
from oracle import paged_attention as opa
from tests.gpu_helpers import (bf16_to_f64, build_tables, compare, default_scale, poison_unused,
                               run_decode)
import workloads

pytestmark = pytest.mark.gpu

VARIANTS = {"auto": pk.PA_DECODE_AUTO, "cuda_core": pk.PA_DECODE_CUDA_CORE, "mma": pk.PA_DECODE_MMA,
            "tcgen05": pk.PA_DECODE_TCGEN05}


def make_case(lens, hq, hkv, d, bs, seed, extra_blocks=4):
    nb = sum(-(-int(n) // bs) for n in lens) + extra_blocks
    rng = np.random.default_rng(seed)
    order = rng.permutation(nb)
    t_ref, l_ref, t_cpp, l_cpp, used = build_tables(lens, bs, nb, order)
    pool = workloads.bf16_normal((nb, 2, hkv, bs, d), seed=seed)
    poison_unused(pool, used)
    q = workloads.bf16_normal((len(lens), hq, d), seed=seed + 1)
    return q, pool, (t_ref, l_ref), (t_cpp, l_cpp)


def check(lens, hq, hkv, d, bs, seed, variant="auto", partition_tokens=0, scale=None):
    scale = default_scale(d) if scale is None else scale
    q, pool, (t_ref, l_ref), (t_cpp, l_cpp) = make_case(lens, hq, hkv, d, bs, seed)
    want = opa.decode(bf16_to_f64(q), bf16_to_f64(pool), t_ref, l_ref, scale)
    out = run_decode(q.cuda(), pool.cuda(), t_cpp, l_cpp, scale, VARIANTS[variant], partition_tokens)
    assert pk.pa_device_error() == 0
    return compare(bf16_to_f64(out), want)


RAGGED = [1, 15, 16, 17, 32, 53, 100, 257, 600]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_auto_variant_ragged(d, bs, group):
    hkv = 2
    check(RAGGED, hkv * group, hkv, d, bs, seed=7 * d + bs + group)


@pytest.mark.parametrize("variant,group", [("cuda_core", 1), ("cuda_core", 2), ("cuda_core", 4),
                                           ("mma", 1), ("mma", 2), ("mma", 3), ("mma", 4), ("mma", 5),
                                           ("mma", 8)])
@pytest.mark.parametrize("d,bs", [(128, 16), (64, 32), (64, 16)])  # 64/16: two blocks per tile
@pytest.mark.parametrize("schedule", [pk.PA_SCHEDULE_BALANCED, 0, 64])
def test_each_variant(variant, group, d, bs, schedule):
    check([5, 31, 33, 200, 480], 2 * group, 2, d, bs, seed=100 + group, variant=variant,
          partition_tokens=schedule)


@pytest.mark.parametrize("partition_blocks", [1, 2, 3, 8, 64])
@pytest.mark.parametrize("variant", ["cuda_core", "mma"])
def test_split_k_partitions(partition_blocks, variant):
    """Many, few and a single partition agree with the oracle (split-K + LSE merge)."""
    bs = 16
    check([1, 16, 47, 300, 1000], 8, 2, 128, bs, seed=55, variant=variant,
          partition_tokens=partition_blocks * bs)


@pytest.mark.parametrize("lens", [
    [1, 0, 3],                 # fewer units than CTAs: most CTAs get nothing
    [0, 0, 0, 0],              # nothing to attend over anywhere
    [40000],                   # one request cut across every CTA
    [17, 40000, 0, 5, 2048],   # mixed, with a request split many ways
])
@pytest.mark.parametrize("variant", ["mma", "cuda_core", "tcgen05", "tcgen05_two_halves"])
def test_balanced_schedule_edges(lens, variant):
    hq, hkv = {"mma": (8, 2), "cuda_core": (4, 4), "tcgen05": (32, 2), "tcgen05_two_halves": (58, 2)}[variant]
    v = "tcgen05" if variant.startswith("tcgen05") else variant
    for d in (64, 128) if v == "tcgen05" else (64,):
        check(lens, hq, hkv, d, 16, seed=60 + len(lens), variant=v, partition_tokens=pk.PA_SCHEDULE_BALANCED)


def test_balanced_matches_partition_grid():
    lens = [3000, 17, 1200, 2049, 5, 640, 2999, 1, 4096, 33]
    q, pool, _, (t, l) = make_case(lens, 32, 8, 128, 16, seed=61)
    q, pool = q.cuda(), pool.cuda()
    bal = run_decode(q, pool, t, l, 0.088, pk.PA_DECODE_MMA, partition_tokens=pk.PA_SCHEDULE_BALANCED)
    grid = run_decode(q, pool, t, l, 0.088, pk.PA_DECODE_MMA, partition_tokens=512)
    assert (bal.float() - grid.float()).abs().max().item() <= 2 ** -7


@pytest.mark.parametrize("d,bs", [(128, 16), (64, 32), (64, 16)])
@pytest.mark.parametrize("schedule", [0, pk.PA_SCHEDULE_BALANCED])
@pytest.mark.parametrize("hq,hkv", [(32, 2), (24, 2), (64, 2), (32, 1)])
@pytest.mark.parametrize("variant", ["auto", "mma"])
def test_wide_groups(d, bs, schedule, hq, hkv, variant):
    """Groups of 12, 16 and 32 query heads per KV head (32/1: multi-query),
    balanced schedule only: by default the tcgen05 consumer; on request
    mma.sync with two or four 8-wide MMA tiles on grouped warps."""
    check(RAGGED, hq, hkv, d, bs, seed=70 + d + bs + hq, variant=variant, partition_tokens=schedule)


@pytest.mark.parametrize("d,bs", [(128, 16), (128, 32), (64, 16), (64, 32)])
@pytest.mark.parametrize("hq,hkv", [(2, 2), (8, 2), (18, 2), (26, 2), (32, 2), (16, 1), (96, 8),
                                    (34, 2), (48, 2), (62, 2), (64, 2), (32, 1), (256, 8)])
def test_tcgen05_variant(d, bs, hq, hkv):
    """The tcgen05 consumer for 1..32 (token, head) columns (one 16-column
    half, or two sharing each tile from 17 columns): 128-token tiles with
    ragged ends, tiles cut between CTAs, requests of exactly one tile, NaN
    in every unused pool row."""
    check(RAGGED + [2000, 129, 128, 127, 4111], hq, hkv, d, bs, seed=300 + d + bs + hq + hkv, variant="tcgen05")


def test_tcgen05_rejects_more_than_32_columns():
    q, pool, _, (t, l) = make_case([40, 70], 68, 2, 128, 16, seed=301)
    with pytest.raises(pk.PaError):
        run_decode(q.cuda(), pool.cuda(), t, l, 0.1, pk.PA_DECODE_TCGEN05)


@pytest.mark.parametrize("hq,hkv", [(24, 2), (32, 2), (48, 2), (64, 2)])
def test_tcgen05_matches_mma_sync(hq, hkv):
    """Both tensor-core consumers on the same wide-group inputs: equal up to
    the rounding of their different summation orders."""
    lens = [3000, 17, 1200, 2049, 5, 640, 2999, 1, 4096, 33]
    q, pool, _, (t, l) = make_case(lens, hq, hkv, 128, 16, seed=64 + hq)
    q, pool = q.cuda(), pool.cuda()
    a = run_decode(q, pool, t, l, 0.088, pk.PA_DECODE_TCGEN05)
    b = run_decode(q, pool, t, l, 0.088, pk.PA_DECODE_MMA, partition_tokens=pk.PA_SCHEDULE_BALANCED)
    assert (a.float() - b.float()).abs().max().item() <= 2 ** -7


def check_short(lens, hq, hkv, d, bs, seed, variant="auto", partition_tokens=pk.PA_SCHEDULE_BALANCED):
    """check() for batches of very short requests (0..~40 positions): an
    output then averages a handful of value rows, so the bf16 rounding of the
    probabilities (relative 2^-9 per weight, 2^-8 after normalising) moves it
    by up to 2^-8 max_pos |v - out|, and the bf16 output by up to 2^-8
    |out|; over the 0.5-1 M outputs of these shapes that can pass 1e-2 with
    no kernel error at all.  Each element is bounded by 1e-2 plus those two
    terms (the spread over the request's own value rows); the mean stays
    <= 1e-3."""
    q, pool, (t_ref, l_ref), (t_cpp, l_cpp) = make_case(lens, hq, hkv, d, bs, seed=seed)
    scale = default_scale(d)
    pool64, q64 = bf16_to_f64(pool), bf16_to_f64(q)
    want = opa.decode(q64, pool64, t_ref, l_ref, scale)
    out = run_decode(q.cuda(), pool.cuda(), t_cpp, l_cpp, scale, VARIANTS[variant], partition_tokens)
    assert pk.pa_device_error() == 0
    got = bf16_to_f64(out)
    g = hq // hkv
    spread = np.zeros_like(want)
    for b, n in enumerate(l_ref):
        if n == 0:
            continue
        rows = np.stack([pool64[t_ref[b][p // bs], 1, :, p % bs, :] for p in range(int(n))])  # [n, hkv, d]
        vmax = np.repeat(rows.max(axis=0), g, axis=0)  # [hq, d]: query head j reads KV head j // g
        vmin = np.repeat(rows.min(axis=0), g, axis=0)
        spread[b] = np.maximum(np.abs(vmax - want[b]), np.abs(vmin - want[b]))
    err = np.abs(got - want)
    assert np.isfinite(got).all()
    bound = 1e-2 + 2.0 ** -8 * (spread + np.abs(want))
    assert (err <= bound).all(), float((err - bound).max())
    assert err.mean() <= 1e-3


@pytest.mark.parametrize("hq,variant", [(8, "mma"), (32, "tcgen05"), (64, "tcgen05")])
def test_balanced_schedule_at_its_batch_limit(hq, variant):
    """4096 requests (the prefix table in shared memory at its largest) on the
    balanced schedule, short ragged lengths including empty requests; the
    tcgen05 consumer with one and with two halves."""
    lens = list(np.random.default_rng(63).integers(0, 40, size=4096))
    check_short(lens, hq, 2, 128, 16, seed=63, variant=variant)


@pytest.mark.parametrize("batch", [512, 513])
@pytest.mark.parametrize("hq,variant", [(8, "mma"), (32, "tcgen05"), (64, "tcgen05")])
def test_merge_prefix_sums_either_side_of_its_local_limit(batch, hq, variant):
    """The merge kernel of the balanced schedule computes the block-count
    prefix sums itself for up to 512 requests and reads the decode kernel's
    copy above that: both sides of the limit, with many (request, head) pairs
    cut between CTAs and some empty requests."""
    lens = list(np.random.default_rng(66 + batch).integers(0, 200, size=batch))
    check_short(lens, hq, 2, 128, 16, seed=66 + batch, variant=variant)


@pytest.mark.parametrize("hq,d,bs", [(32, 128, 16), (32, 64, 16), (48, 128, 32)])
def test_wide_groups_above_the_batch_limit(hq, d, bs):
    """More than 8 columns with more than 4096 requests: the default variant
    runs the tcgen05 consumer (its prefix table lives in the tile ring), at
    head dim 64 too; mma.sync is refused."""
    lens = list(np.random.default_rng(64).integers(0, 30, size=4200))
    check_short(lens, hq, 2, d, bs, seed=64, variant="auto", partition_tokens=0)
    q, pool, _, (t, l) = make_case(lens[:4200], hq, 2, d, bs, seed=65)
    with pytest.raises(pk.PaError):
        run_decode(q.cuda(), pool.cuda(), t, l, 0.1, pk.PA_DECODE_MMA, pk.PA_SCHEDULE_BALANCED)


def test_batch_above_balanced_limit_uses_grid():
    lens = list(np.random.default_rng(62).integers(0, 40, size=4100))
    check(lens, 4, 2, 64, 16, seed=62)


def test_split_k_consistency():
    """P=1 and P>1 results agree to fp32-merge rounding, not just to the tolerance."""
    lens = [700, 1024, 64]
    q, pool, _, (t, l) = make_case(lens, 16, 4, 128, 16, seed=9)
    q, pool = q.cuda(), pool.cuda()
    one = run_decode(q, pool, t, l, 0.088, pk.PA_DECODE_MMA, partition_tokens=2048)
    many = run_decode(q, pool, t, l, 0.088, pk.PA_DECODE_MMA, partition_tokens=64)
    diff = (one.float() - many.float()).abs().max().item()
    assert diff <= 2 ** -7, diff


def test_cuda_core_and_mma_agree():
    lens = [333, 90, 1500]
    q, pool, _, (t, l) = make_case(lens, 8, 2, 128, 16, seed=10)
    q, pool = q.cuda(), pool.cuda()
    a = run_decode(q, pool, t, l, 0.1, pk.PA_DECODE_CUDA_CORE)
    b = run_decode(q, pool, t, l, 0.1, pk.PA_DECODE_MMA)
    assert (a.float() - b.float()).abs().max().item() <= 1e-2


def test_length_one_returns_v():
    """A request of length 1 attends to one token: out equals V exactly."""
    lens = [1, 1, 1]
    q, pool, (t_ref, _), (t, l) = make_case(lens, 8, 2, 128, 16, seed=11)
    for variant in (pk.PA_DECODE_CUDA_CORE, pk.PA_DECODE_MMA):
        out = run_decode(q.cuda(), pool.cuda(), t, l, 0.3, variant).cpu()
        for b in range(3):
            for j in range(8):
                assert torch.equal(out[b, j], pool[t_ref[b, 0], 1, j // 4, 0])


def test_zero_length_request():
    lens = [0, 40, 0, 7]
    q, pool, (t_ref, l_ref), (t, l) = make_case(lens, 4, 4, 64, 16, seed=12)
    out = run_decode(q.cuda(), pool.cuda(), t, l, 0.125).cpu()
    assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[2]) == 0
    want = opa.decode(bf16_to_f64(q), bf16_to_f64(pool), t_ref, l_ref, 0.125)
    compare(bf16_to_f64(out), want)


@pytest.mark.parametrize("lens,hq,hkv,d,bs,seed,variant", [
    ([77, 500], 8, 2, 128, 16, 13, "auto"),
    ([77, 500], 4, 4, 64, 16, 14, "auto"),
    ([77, 500, 3000], 32, 2, 128, 16, 15, "tcgen05"),
    ([77, 500, 3000], 24, 2, 64, 32, 16, "tcgen05"),
    ([77, 500, 3000], 64, 2, 128, 16, 17, "tcgen05"),
    ([77, 500, 3000], 40, 2, 64, 16, 18, "tcgen05"),
    ([77, 500, 3000], 64, 2, 128, 16, 17, "mma"),
])
def test_large_logits(lens, hq, hkv, d, bs, seed, variant):
    """Scale 4 (45x the usual 1/sqrt(128)) makes the softmax nearly one-hot;
    the online max must hold (for the wide groups: the column maxima and the
    rescale of O in tensor memory).  An output is then nearly one value
    row, up to ~4.5 in magnitude, and its bf16 rounding alone can reach half
    a unit in the last place, 2^-8 |out| (0.0176 at 4.5): so here the bound
    per element is 1e-2 + 2^-8 |want| (the fixed 1e-2 plus that rounding),
    and the mean stays <= 1e-3."""
    q, pool, (t_ref, l_ref), (t_cpp, l_cpp) = make_case(lens, hq, hkv, d, bs, seed)
    want = opa.decode(bf16_to_f64(q), bf16_to_f64(pool), t_ref, l_ref, 4.0)
    out = run_decode(q.cuda(), pool.cuda(), t_cpp, l_cpp, 4.0, VARIANTS[variant],
                     pk.PA_SCHEDULE_BALANCED if hq // hkv > 8 else 0)
    assert pk.pa_device_error() == 0
    got = bf16_to_f64(out)
    err = np.abs(got - want)
    assert np.isfinite(got).all()
    assert (err <= 1e-2 + 2.0 ** -8 * np.abs(want)).all(), float((err - 2.0 ** -8 * np.abs(want)).max())
    assert err.mean() <= 1e-3


def test_tiny_workload():
    """The tiny workload end to end: lengths U[1,64], one appended token."""
    p = workloads.plan("tiny")
    s = p.shape
    lens = [int(n) + 1 for n in p.seq_lens]
    check(lens, s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size, seed=workloads.seed_of("tiny"))


def test_device_checks_flag_bad_inputs():
    """Bad block ids / lengths are flagged, skipped or clamped; nothing faults."""
    lens = [40, 40]
    q, pool, _, (t, l) = make_case(lens, 4, 2, 128, 16, seed=15)
    q, pool = q.cuda(), pool.cuda()
    pk.pa_device_error(clear=True)
    bad = t.copy()
    bad[0, 1] = pool.shape[0] + 5
    run_decode(q, pool, bad, l, 0.1)
    assert pk.pa_device_error() & pk.PA_DEVERR_BLOCK_ID
    long_lens = l.copy()
    long_lens[1] = t.shape[1] * 16 + 9  # beyond the table row
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    pk.pa_decode(out, q, pool, torch.as_tensor(t, device="cuda"), torch.as_tensor(long_lens, device="cuda"),
                 int(long_lens.max()), 0.1, workspace=ws)
    torch.cuda.synchronize()
    assert pk.pa_device_error() & pk.PA_DEVERR_SEQ_LEN
    assert pk.pa_device_error() == 0  # cleared by the previous read


BAD_ID_CASES = [(v, 128, 16, pk.PA_SCHEDULE_BALANCED, 8) for v in ("mma", "cuda_core", "tcgen05")] + \
    [(v, 128, 16, 64, 8) for v in ("mma", "cuda_core")] + \
    [(v, 64, 16, pk.PA_SCHEDULE_BALANCED, 8) for v in ("mma", "cuda_core", "tcgen05")] + \
    [(v, 64, 32, 0, 8) for v in ("mma", "cuda_core", "tcgen05")] + \
    [(v, d, 16, pk.PA_SCHEDULE_BALANCED, 40) for v in ("mma", "tcgen05") for d in (64, 128)]


@pytest.mark.parametrize("variant,d,bs,schedule,hq", BAD_ID_CASES)
def test_bad_block_ids_read_zeros(variant, d, bs, schedule, hq):
    """A table entry outside [0, num_blocks) -- past the end or negative --
    reads a block of zeros and flags PA_DEVERR_BLOCK_ID: the output equals the
    oracle's over a pool whose extra block is all zeros.  (Group 20: the
    paired-warp mma.sync kernel and the tcgen05 consumer's two halves.)"""
    lens = [40, 100, 70]
    q, pool, (t_ref, l_ref), (t, l) = make_case(lens, hq, 2, d, bs, seed=17 + d + bs)
    nb = pool.shape[0]
    bad = t.copy()
    bad[0, 1] = nb + 5
    bad[1, 0] = -3
    bad[2, (70 - 1) // bs] = nb  # the ragged last block
    zero_pool = torch.cat([pool, torch.zeros((1,) + tuple(pool.shape[1:]), dtype=pool.dtype)])
    t_zero = t_ref.copy()
    t_zero[0, 1] = t_zero[1, 0] = t_zero[2, (70 - 1) // bs] = nb
    want = opa.decode(bf16_to_f64(q), bf16_to_f64(zero_pool), t_zero, l_ref, default_scale(d))
    pk.pa_device_error(clear=True)
    out = run_decode(q.cuda(), pool.cuda(), bad, l, default_scale(d), VARIANTS[variant], schedule)
    assert pk.pa_device_error() == pk.PA_DEVERR_BLOCK_ID
    compare(bf16_to_f64(out), want)


def test_wait_timeout_is_reported():
    pk.pa_device_error(clear=True)
    pk.pa_selftest_wait_timeout(20_000_000)  # 20 ms
    torch.cuda.synchronize()
    assert pk.pa_device_error() == pk.PA_DEVERR_WAIT_TIMEOUT
    # the context is still usable
    check([20], 4, 4, 64, 16, seed=16)
