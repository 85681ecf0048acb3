"""pa_decode_multi (T causal query tokens per request) against the fp64 oracle.

Query token t of request b sits at position L_b - T + t and attends to
[0, L_b - T + t].  Unused pool rows are NaN; requests shorter than T, T = 1
(which must match pa_decode) and the widest tile (group x T = 16) are
covered.
"""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_354_b200 as pk
import workloads
from oracle import paged_attention as opa
from tests.gpu_helpers import bf16_to_f64, build_tables, compare, poison_unused, run_decode

pytestmark = pytest.mark.gpu


def make(lens, T, hq, hkv, d, bs, seed):
    nb = sum(-(-int(n) // bs) for n in lens) + 4
    order = np.random.default_rng(seed).permutation(nb)
    t_ref, l_ref, t_cpp, l_cpp, used = build_tables(lens, bs, nb, order)
    pool = poison_unused(workloads.bf16_normal((nb, 2, hkv, bs, d), seed=seed), used)
    q = workloads.bf16_normal((len(lens), T, hq, d), seed=seed + 1)
    return q, pool, (t_ref, l_ref), (t_cpp, l_cpp)


def run_multi(q, pool, tables, lens, scale):
    b, T, hq, d = q.shape
    hkv, bs = pool.shape[2], pool.shape[3]
    max_len = max(1, int(np.max(lens)))
    ws = torch.empty(max(256, pk.pa_decode_multi_workspace_size(b, T, hq, hkv, d, bs, max_len)),
                     dtype=torch.uint8, device="cuda")
    out = torch.full_like(q, float("nan"))
    pk.pa_decode_multi(out, q, pool, torch.as_tensor(tables, device="cuda"), torch.as_tensor(lens, device="cuda"),
                       max_len, scale, ws)
    torch.cuda.synchronize()
    return out


# columns per KV head (group x T): 4, 16, 16, 16, 16, 9, 5, 12, 15, 32, 21,
# 24, 32 -- at head dim 128, 9 to 32 the tcgen05 consumer (one or two
# 16-column halves); up to 8, and at head dim 64, the mma.sync consumer
@pytest.mark.parametrize("T,hq,hkv", [(2, 8, 2), (4, 8, 2), (8, 4, 2), (2, 16, 2), (16, 2, 2), (3, 12, 4), (5, 4, 4),
                                      (3, 8, 2), (3, 10, 2), (4, 16, 2), (3, 14, 2), (3, 16, 2), (2, 32, 2)])
@pytest.mark.parametrize("d,bs", [(128, 16), (64, 32), (64, 16)])
def test_multi_matches_oracle(T, hq, hkv, d, bs):
    lens = [T, T + 1, 17, 33, 250, 1000, 2049]
    q, pool, (t_ref, l_ref), (t, l) = make(lens, T, hq, hkv, d, bs, seed=200 + T + hq)
    scale = 1.0 / math.sqrt(d)
    want = opa.decode_multi(bf16_to_f64(q), bf16_to_f64(pool), t_ref, l_ref, scale)
    got = run_multi(q.cuda(), pool.cuda(), t, l, scale)
    assert pk.pa_device_error() == 0
    compare(bf16_to_f64(got), want)


def test_multi_short_requests_get_zero():
    lens = [1, 2, 0, 5]
    T = 4
    q, pool, (t_ref, l_ref), (t, l) = make(lens, T, 8, 2, 128, 16, seed=210)
    got = run_multi(q.cuda(), pool.cuda(), t, l, 0.1).cpu()
    want = opa.decode_multi(bf16_to_f64(q), bf16_to_f64(pool), t_ref, l_ref, 0.1)
    assert torch.count_nonzero(got[0, :3]) == 0 and torch.count_nonzero(got[2]) == 0
    compare(bf16_to_f64(got), want)


def test_single_token_matches_pa_decode():
    lens = [5, 300, 1200, 64]
    q, pool, _, (t, l) = make(lens, 1, 32, 8, 128, 16, seed=211)
    q, pool = q.cuda(), pool.cuda()
    multi = run_multi(q, pool, t, l, 0.09)[:, 0]
    single = run_decode(q[:, 0].contiguous(), pool, t, l, 0.09, pk.PA_DECODE_MMA, pk.PA_SCHEDULE_BALANCED)
    assert torch.equal(multi, single)


def test_multi_rejects_too_wide_tiles():
    with pytest.raises(pk.PaError):
        pk.pa_decode_multi_workspace_size(4, 3, 96, 8, 128, 16, 100)  # group 12 x 3 tokens = 36 columns


def test_multi_above_the_batch_limit():
    """4200 requests, 2 query tokens x group 8 (16 columns): the tcgen05
    consumer, whose prefix table takes batches above 4096."""
    lens = [int(x) for x in np.random.default_rng(66).integers(0, 24, size=4200)]
    T, hq, hkv, d, bs = 2, 16, 2, 128, 16
    q, pool, (t_ref, l_ref), (t, l) = make(lens, T, hq, hkv, d, bs, seed=66)
    scale = 1.0 / math.sqrt(d)
    want = opa.decode_multi(bf16_to_f64(q), bf16_to_f64(pool), t_ref, l_ref, scale)
    got = bf16_to_f64(run_multi(q.cuda(), pool.cuda(), t, l, scale))
    assert pk.pa_device_error() == 0
    # very short requests: the bf16 probabilities and output can move an
    # element by 2^-8 (|v - out| spread + |out|) beyond the 1e-2 bound (see
    # tests/test_gpu_decode.py, check_short); with |v| < ~5.5 that is < 0.065
    err = np.abs(got - want)
    assert np.isfinite(got).all() and err.mean() <= 1e-3
    assert (err <= 1e-2 + 2.0 ** -8 * (11.0 + np.abs(want))).all()
