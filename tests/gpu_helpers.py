"""Shared helpers for the GPU parity tests (test-side marshalling only)."""

import math

import numpy as np
import torch

import paged_kv_cache_354_b200 as pk
import workloads
from oracle.block_allocator import BlockAllocator

MAX_ABS = 1e-2  # attention outputs vs the fp64 oracle: max |err|
MEAN_ABS = 1e-3  # and mean |err|


def bf16_to_f64(t):
    """Exact float64 values of a bf16 tensor (CPU numpy)."""
    return t.detach().to("cpu", torch.float32).double().numpy()


def u16_to_f64(a):
    """Exact float64 values of bf16 bit patterns held as uint16."""
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_nan():
    return torch.tensor(float("nan"), dtype=torch.bfloat16)


def build_tables(lens, bs, num_blocks, order):
    """Fill requests 0..B-1 to `lens` with both allocators.

    Returns (oracle tables, oracle lens, C++ tables, C++ lens, used slots);
    the oracle side never sees the C++ result.
    """
    ref = BlockAllocator(num_blocks, bs, order)
    cpp = pk.PaAlloc(num_blocks, bs, order)
    used = []
    for i, n in enumerate(lens):
        ref.add_seq(i)
        cpp.add_seq(i)
        if n:
            used += ref.append(i, int(n))[0]
            cpp.append(i, int(n))
    ids = list(range(len(lens)))
    mb = max(1, max(-(-int(n) // bs) for n in lens))
    t_ref, l_ref = workloads.block_tables(ref, ids, mb)
    t_cpp, l_cpp = cpp.block_tables(ids, mb)
    return t_ref, l_ref, t_cpp, l_cpp, used


def poison_unused(pool, used_slots):
    """Set every pool row that holds no request's token to NaN."""
    nb, _, _, bs, _ = pool.shape
    keep = torch.zeros(nb * bs, dtype=torch.bool)
    keep[torch.as_tensor(used_slots, dtype=torch.long)] = True
    mask = (~keep).view(nb, 1, 1, bs, 1).expand_as(pool)
    pool[mask] = bf16_nan()
    return pool


def compare(got, want, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - want)
    assert np.isfinite(got).all(), "non-finite output"
    assert err.max() <= max_abs, f"max abs err {err.max():.3e} > {max_abs}"
    assert err.mean() <= mean_abs, f"mean abs err {err.mean():.3e} > {mean_abs}"
    return float(err.max()), float(err.mean())


def workspace_for(batch, hq, hkv, d, bs, max_seq_len, partition_tokens=0):
    nbytes, parts = pk.pa_decode_workspace_size(batch, hq, hkv, d, bs, max_seq_len, partition_tokens)
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda"), parts


def run_decode(q, pool, tables, lens, scale, variant=pk.PA_DECODE_AUTO, partition_tokens=0):
    b, hq, d = q.shape
    hkv, bs = pool.shape[2], pool.shape[3]
    max_len = int(max(1, int(lens.max()) if len(lens) else 1))
    # the tcgen05 consumer always runs the balanced schedule: size for it
    ws_schedule = pk.PA_SCHEDULE_BALANCED if variant == pk.PA_DECODE_TCGEN05 else partition_tokens
    ws, _ = workspace_for(b, hq, hkv, d, bs, max_len, ws_schedule)
    out = torch.full_like(q, float("nan"))
    pk.pa_decode(out, q, pool, torch.as_tensor(tables, device="cuda"), torch.as_tensor(lens, device="cuda"),
                 max_len, scale, workspace=ws, variant=variant, partition_tokens=partition_tokens)
    torch.cuda.synchronize()
    return out


def default_scale(d):
    return 1.0 / math.sqrt(d)
