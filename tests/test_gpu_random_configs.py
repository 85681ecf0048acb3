"""Seeded random configurations of pa_decode and pa_decode_multi against the
fp64 oracle: batch, lengths (0 included), KV heads, group, query tokens,
head dim, block size, consumer and schedule all drawn per case, so shapes
that no hand-written case names (odd groups, a tcgen05 half that is mostly
padding, short batches on the balanced schedule) get covered.  Unused pool
rows are NaN.  Tolerance: max |err| <= 1e-2, mean <= 1e-3."""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_354_b200 as pk
import workloads
from oracle import paged_attention as opa
from tests.gpu_helpers import bf16_to_f64, build_tables, compare, poison_unused

pytestmark = pytest.mark.gpu

VARIANTS = [pk.PA_DECODE_AUTO, pk.PA_DECODE_MMA, pk.PA_DECODE_TCGEN05, pk.PA_DECODE_CUDA_CORE]


def draw(seed):
    rng = np.random.default_rng(seed)
    d = int(rng.choice([64, 128]))
    bs = int(rng.choice([16, 32]))
    hkv = int(rng.integers(1, 5))
    T = int(rng.choice([1, 1, 1, 2, 3, 4]))
    g = int(rng.integers(1, 32 // T + 1))
    batch = int(rng.integers(1, 13))
    lens = [int(x) for x in rng.integers(0, 3000, size=batch)]
    if rng.random() < 0.5:  # one request shorter than T, possibly empty
        lens[int(rng.integers(batch))] = int(rng.integers(0, T + 1))
    variant = int(rng.choice(VARIANTS))
    if variant == pk.PA_DECODE_CUDA_CORE and (g not in (1, 2, 4) or T > 1):
        variant = pk.PA_DECODE_MMA
    balanced = T > 1 or g > 8 or variant == pk.PA_DECODE_TCGEN05 or rng.random() < 0.5
    return dict(d=d, bs=bs, hkv=hkv, g=g, T=T, lens=lens, variant=variant, balanced=balanced)


@pytest.mark.parametrize("seed", range(100))
def test_random_configuration(seed):
    c = draw(9000 + seed)
    d, bs, hkv, g, T, lens = c["d"], c["bs"], c["hkv"], c["g"], c["T"], c["lens"]
    hq = hkv * g
    nb = sum(-(-n // bs) for n in lens) + 3
    order = np.random.default_rng(seed).permutation(nb)
    t_ref, l_ref, t_cpp, l_cpp, used = build_tables(lens, bs, nb, order)
    pool = poison_unused(workloads.bf16_normal((nb, 2, hkv, bs, d), seed=seed + 1), used)
    scale = 1.0 / math.sqrt(d)
    max_len = max(1, max(lens))
    dev = torch.device("cuda")
    tables, seq_lens, gpool = torch.as_tensor(t_cpp, device=dev), torch.as_tensor(l_cpp, device=dev), pool.to(dev)
    pk.pa_device_error(clear=True)
    if T == 1:
        q = workloads.bf16_normal((len(lens), hq, d), seed=seed + 2)
        want = opa.decode(bf16_to_f64(q), bf16_to_f64(pool), t_ref, l_ref, scale)
        sched = pk.PA_SCHEDULE_BALANCED if c["balanced"] else 0
        nbytes, _ = pk.pa_decode_workspace_size(len(lens), hq, hkv, d, bs, max_len, sched)
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
        out = torch.full_like(q.to(dev), float("nan"))
        pk.pa_decode(out, q.to(dev), gpool, tables, seq_lens, max_len, scale, workspace=ws, variant=c["variant"],
                     partition_tokens=sched)
    else:
        q = workloads.bf16_normal((len(lens), T, hq, d), seed=seed + 2)
        want = opa.decode_multi(bf16_to_f64(q), bf16_to_f64(pool), t_ref, l_ref, scale)
        ws = torch.empty(max(256, pk.pa_decode_multi_workspace_size(len(lens), T, hq, hkv, d, bs, max_len)),
                         dtype=torch.uint8, device=dev)
        out = torch.full_like(q.to(dev), float("nan"))
        pk.pa_decode_multi(out, q.to(dev), gpool, tables, seq_lens, max_len, scale, ws)
    torch.cuda.synchronize()
    assert pk.pa_device_error() == 0, c
    compare(bf16_to_f64(out), want)
