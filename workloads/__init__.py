"""Seeded synthetic inputs for the five paged-decode workloads.

This module is shared by the tests, the oracle runs and the benchmark.  It
holds none of the method's arithmetic: it draws random numbers (sequence
lengths, a shuffled free-list order, churn events, bf16 N(0,1) tensors) and
drives *an* allocator through its public calls.  Block tables and slot
mappings always come from the allocator under test (the C++ one for the
product path, the Python model for the oracle path), never from here.

Workloads (seed = 354 + index in ``NAMES``):

tiny     B4, Hq=Hkv=4, D64, bs16, 64 blocks; lengths U[1,64]; one appended
         token per request.
llama8b  Llama-3-8B decode shape: B64, Hq32/Hkv8 (GQA group 4), D128, bs16;
         lengths U[512,4096]; pool 1.1x the blocks needed, shuffled.
long     split-K stress: B4, length 32768 each, Hq32/Hkv8, D128, bs16; the
         pool is exactly the blocks needed, shuffled.
beam     prefix sharing + copy-on-write: 8 prompts x 4 beams, Hq64/Hkv8
         (group 8), D128, bs16; a 2050-token prefix per prompt shared by its
         4 beams, then 256 divergent tokens per beam.
mixed    serving step: B256, Hq32/Hkv8, D128, bs32; lengths lognormal
         (median 1024, sigma 1) clipped to [1, 8192]; the pool is fragmented
         by 1000 seeded alloc/free churn events; one appended token each.
"""

from dataclasses import dataclass
import math

import numpy as np

NAMES = ("tiny", "llama8b", "long", "beam", "mixed")
SEED_BASE = 354


def seed_of(name):
    return SEED_BASE + NAMES.index(name)


@dataclass(frozen=True)
class Shape:
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int


SHAPES = {
    "tiny": Shape("tiny", 4, 4, 64, 16),
    "llama8b": Shape("llama8b", 32, 8, 128, 16),
    "long": Shape("long", 32, 8, 128, 16),
    "beam": Shape("beam", 64, 8, 128, 16),
    "mixed": Shape("mixed", 32, 8, 128, 32),
}


def _blocks_for(tokens, block_size):
    return -(-int(tokens) // block_size)


# --------------------------------------------------------------------------
# random draws
# --------------------------------------------------------------------------
def rng(name, stream=0):
    """numpy Generator for a workload; ``stream`` separates independent draws."""
    return np.random.default_rng([seed_of(name), stream])


def shuffled_order(num_blocks, gen):
    """A random permutation of the physical blocks (initial free-list order)."""
    return gen.permutation(num_blocks).astype(np.int64)


def bf16_normal(shape, seed, device="cpu"):
    """bf16 tensor: float32 N(0,1) from a seeded torch generator, rounded RNE."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def lengths(name, gen, batch=None):
    """Draw the request lengths of a workload (before any appended token)."""
    if name == "tiny":
        return gen.integers(1, 64, size=batch or 4, endpoint=True)
    if name == "llama8b":
        return gen.integers(512, 4096, size=batch or 64, endpoint=True)
    if name == "long":
        return np.full(batch or 4, 32768, dtype=np.int64)
    if name == "mixed":
        raw = gen.lognormal(mean=math.log(1024.0), sigma=1.0, size=batch or 256)
        return np.clip(np.rint(raw), 1, 8192).astype(np.int64)
    raise ValueError(name)


# --------------------------------------------------------------------------
# allocator drivers (work with any object exposing the allocator calls)
# --------------------------------------------------------------------------
@dataclass
class Plan:
    """Everything needed to build the same allocator state twice."""

    name: str
    shape: Shape
    num_blocks: int
    initial_order: np.ndarray
    seq_lens: np.ndarray  # lengths the requests are filled to before the append
    append_tokens: int  # tokens appended to every request in the hot-path step
    beams: int = 0
    prefix_len: int = 0


def plan(name, batch=None, extra_tokens=0):
    """Draw the lengths and pool order of a workload.

    ``extra_tokens`` reserves room in the pool for that many further tokens
    per request (the benchmark appends one token per request per step).
    """
    shape = SHAPES[name]
    bs = shape.block_size
    gen = rng(name)
    if name == "beam":
        prompts, beams, prefix, grow = 8, 4, 2050, 256
        need = prompts * _blocks_for(prefix, bs) + prompts * beams * (
            _blocks_for(prefix + grow + extra_tokens, bs) - _blocks_for(prefix, bs) + 1
        )
        num_blocks = int(math.ceil(1.1 * need))
        order = shuffled_order(num_blocks, gen)
        return Plan(name, shape, num_blocks, order, np.full(prompts, prefix), grow,
                    beams=beams, prefix_len=prefix)
    lens = lengths(name, gen, batch)
    append = 1 if name in ("tiny", "mixed") else 0
    need = sum(_blocks_for(L + append + extra_tokens, bs) for L in lens)
    if name == "tiny":
        num_blocks = max(64, need)
    elif name == "llama8b":
        num_blocks = int(math.ceil(1.1 * need))
    elif name == "long":
        num_blocks = need
    elif name == "mixed":
        num_blocks = int(math.ceil(1.25 * need)) + 64
    order = shuffled_order(num_blocks, gen)
    return Plan(name, shape, num_blocks, order, lens.astype(np.int64), append)


def churn(alloc, name, events=1000, first_id=1_000_000):
    """Seeded alloc/free churn that leaves the free list permuted.

    Each event, with probability 1/2 (always, if nothing temporary is
    live), takes a temporary request of U[1,64] blocks if that many are free,
    and otherwise drops a random live temporary request.  All temporaries are
    dropped at the end.
    """
    gen = rng(name, stream=1)
    bs = alloc.block_size
    live = []
    next_id = first_id
    for _ in range(events):
        want_alloc = (not live) or gen.random() < 0.5
        nblk = int(gen.integers(1, 64, endpoint=True))
        if want_alloc and alloc.num_free() >= nblk:
            alloc.add_seq(next_id)
            alloc.append(next_id, nblk * bs)
            live.append(next_id)
            next_id += 1
        elif live:
            victim = live.pop(int(gen.integers(0, len(live))))
            alloc.free_seq(victim)
    for sid in live:
        alloc.free_seq(sid)


def populate(alloc, p):
    """Fill the requests of plan ``p`` (no appended token yet).

    Returns the request ids in batch order.  For ``beam`` the prompt
    requests are filled, forked into beams and dropped, so each prefix block
    ends with one reference per beam; the returned ids are the beams.
    """
    if p.name == "mixed":
        churn(alloc, p.name)
    if p.name == "beam":
        beam_ids = []
        for prompt in range(len(p.seq_lens)):
            pid = 10_000 + prompt
            alloc.add_seq(pid)
            alloc.append(pid, int(p.seq_lens[prompt]))
        for prompt in range(len(p.seq_lens)):
            pid = 10_000 + prompt
            for beam in range(p.beams):
                bid = prompt * p.beams + beam
                alloc.fork(pid, bid)
                beam_ids.append(bid)
        for prompt in range(len(p.seq_lens)):
            alloc.free_seq(10_000 + prompt)
        return beam_ids
    ids = list(range(len(p.seq_lens)))
    for sid in ids:
        alloc.add_seq(sid)
        alloc.append(sid, int(p.seq_lens[sid]))
    return ids


def block_tables(alloc, seq_ids, max_blocks=None):
    """Padded int32 [B, max_blocks] table and int32 lengths, read from ``alloc``."""
    tables = [alloc.block_table(s) for s in seq_ids]
    width = max_blocks or max(1, max(len(t) for t in tables))
    out = np.zeros((len(seq_ids), width), dtype=np.int32)
    for i, t in enumerate(tables):
        out[i, : len(t)] = t
    lens = np.array([alloc.seq_len(s) for s in seq_ids], dtype=np.int32)
    return out, lens
