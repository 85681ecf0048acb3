"""fp64 oracle of the paged-KV data path -- test infrastructure only.

Layout (one pool per layer): ``kv_pool[num_blocks, 2, num_kv_heads,
block_size, head_dim]``; index 0 on the second axis holds keys, 1 holds
values.  The quiz page's sketch ("Conceptual: PagedAttention block lookup")
prints the pool as ``[num_blocks, 2, num_layers, num_kv_heads, block_size,
d_head]``; here the layer axis is dropped because each layer owns its own
pool (a caller loops over layers).  Within a (block, k/v, head) the
``block_size x head_dim`` tile is contiguous in both readings.

Every array is float64; callers pass the exact values of their bf16 inputs
upcast to float64.  Nothing here tiles, splits the sequence, or runs an
online softmax: the gather is the sketch's formula and the attention is the
textbook one, so it shares no algorithm with the CUDA path.
"""

import numpy as np


def reshape_and_cache(kv_pool, key, value, slot_mapping):
    """Write each new token's K/V into the pool slot given by ``slot_mapping``.

    Follows "Paged attention in LLMs", section "The cache being stored" (the
    cache grows by one token's keys and values each step) together with the
    quiz page's sketch, which addresses a token by physical block
    ``slot // block_size`` and in-block offset ``slot % block_size``.

    kv_pool : float64 [NB, 2, Hkv, bs, D], updated in place and returned.
    key, value : float64 [T, Hkv, D]
    slot_mapping : int [T]; a negative slot means "no write" (padding).
    Tokens are written in order t = 0, 1, ..., so a repeated slot keeps the
    last token written to it.
    """
    block_size = kv_pool.shape[3]
    for t in range(len(slot_mapping)):
        slot = int(slot_mapping[t])
        if slot < 0:
            continue
        block, offset = slot // block_size, slot % block_size
        kv_pool[block, 0, :, offset, :] = key[t]
        kv_pool[block, 1, :, offset, :] = value[t]
    return kv_pool


def copy_blocks(kv_pool, block_pairs):
    """Copy whole physical blocks: ``pool[dst] = pool[src]`` for each pair.

    This is the data movement behind the quiz page's comparison table row
    "Beam search / best of N: copy on write blocks": a block shared by several
    requests is duplicated before one of them writes into it.  Pairs are
    applied in order; each copies all of ``[2, Hkv, bs, D]`` (keys and values
    of every head).
    """
    for src, dst in block_pairs:
        kv_pool[int(dst)] = kv_pool[int(src)].copy()
    return kv_pool


def gather_kv(kv_pool, block_table_row, seq_len):
    """Gather one request's keys and values in logical order.

    The quiz page's sketch: for each logical position ``pos`` in
    ``[0, seq_len)`` the physical block is ``block_table[pos // block_size]``
    and the row inside it is ``pos % block_size``.  "Paged attention in LLMs",
    section "Keeping track: the block table": the sequence reads in order
    even though the blocks are scattered.

    Returns (keys, values), each float64 [seq_len, Hkv, D].
    """
    block_size = kv_pool.shape[3]
    pos = np.arange(seq_len)
    phys = np.asarray(block_table_row)[pos // block_size]
    offset = pos % block_size
    keys = kv_pool[phys, 0, :, offset, :]
    values = kv_pool[phys, 1, :, offset, :]
    return keys, values


def decode(query, kv_pool, block_tables, seq_lens, scale):
    """Single-token decode attention over the paged cache, in float64.

    For request b and query head j, with KV head h = j // g where
    g = Hq / Hkv (query heads are grouped onto KV heads in contiguous runs;
    the pages show one head group only, so this grouping is a stated
    reading), gather K_b, V_b through the block table (``gather_kv``) and
    compute the "standard scaled dot product attention" of the sketch:

        s[pos] = scale * sum_d q[b, j, d] * K_b[pos, h, d]
        w      = softmax(s)            (max-subtracted, then normalised)
        out[b, j, :] = sum_pos w[pos] * V_b[pos, h, :]

    A request of length 0 attends over nothing; its output is defined as 0.

    query : float64 [B, Hq, D]; kv_pool : float64 [NB, 2, Hkv, bs, D]
    block_tables : int [B, max_blocks]; seq_lens : int [B]
    Returns float64 [B, Hq, D].
    """
    batch, num_q_heads, head_dim = query.shape
    num_kv_heads = kv_pool.shape[2]
    group = num_q_heads // num_kv_heads
    out = np.zeros((batch, num_q_heads, head_dim), dtype=np.float64)
    for b in range(batch):
        seq_len = int(seq_lens[b])
        if seq_len == 0:
            continue
        keys, values = gather_kv(kv_pool, block_tables[b], seq_len)
        for j in range(num_q_heads):
            h = j // group
            logits = scale * (keys[:, h, :] @ query[b, j])
            weights = np.exp(logits - logits.max())
            weights /= weights.sum()
            out[b, j] = weights @ values[:, h, :]
    return out


def decode_one(query_vec, kv_pool, block_table_row, seq_len, kv_head, scale):
    """Output of one (request, query head) pair; same definition as ``decode``.

    Used where a full-size batch is too large for the oracle and parity is
    checked on sampled (request, head) pairs.
    """
    if seq_len == 0:
        return np.zeros(kv_pool.shape[4], dtype=np.float64)
    keys, values = gather_kv(kv_pool, block_table_row, seq_len)
    logits = scale * (keys[:, kv_head, :] @ query_vec)
    weights = np.exp(logits - logits.max())
    weights /= weights.sum()
    return weights @ values[:, kv_head, :]


def decode_contiguous(query, kv_cache, seq_lens, scale):
    """Single-token decode over a contiguous per-request cache, in float64.

    The layout paging replaces: the quiz page's comparison table, column
    "Naive contiguous allocation", reserves a buffer of the maximum context
    for every request; "Paged attention in LLMs", section "Why the memory
    gets wasted", reserves that maximum up front in one unbroken run.  Here
    request b's run is ``kv_cache[b]`` = [2, Hkv, max_len, D] (keys, then
    values) and positions [0, L_b) of it hold the request's cache.  The
    attention is the same textbook one as ``decode``, with no table.

    query : float64 [B, Hq, D]; kv_cache : float64 [B, 2, Hkv, max_len, D]
    seq_lens : int [B]; returns float64 [B, Hq, D] (0 for L_b = 0).
    """
    batch, num_q_heads, head_dim = query.shape
    num_kv_heads = kv_cache.shape[2]
    group = num_q_heads // num_kv_heads
    out = np.zeros((batch, num_q_heads, head_dim), dtype=np.float64)
    for b in range(batch):
        seq_len = int(seq_lens[b])
        for j in range(num_q_heads if seq_len > 0 else 0):
            keys = kv_cache[b, 0, j // group, :seq_len]
            values = kv_cache[b, 1, j // group, :seq_len]
            logits = scale * (keys @ query[b, j])
            weights = np.exp(logits - logits.max())
            weights /= weights.sum()
            out[b, j] = weights @ values
    return out


def decode_multi(query, kv_pool, block_tables, seq_lens, scale):
    """T query tokens per request, each attending causally (float64).

    The T newest tokens of request b are its queries: token t sits at
    position L_b - T + t (its keys and values are already in the cache) and
    attends to positions [0, L_b - T + t] -- the same gather and softmax as
    ``decode`` over a prefix of the request.  This is the multi-token form a
    speculative-verification or chunked decode step needs; the pages give
    the single-token form, and a query token with no position to attend to
    (L_b - T + t < 0) gets 0 like an empty request.

    query : float64 [B, T, Hq, D]; returns float64 [B, T, Hq, D].
    """
    batch, tokens, num_q_heads, head_dim = query.shape
    num_kv_heads = kv_pool.shape[2]
    group = num_q_heads // num_kv_heads
    out = np.zeros((batch, tokens, num_q_heads, head_dim), dtype=np.float64)
    for b in range(batch):
        for t in range(tokens):
            visible = int(seq_lens[b]) - tokens + t + 1
            if visible <= 0:
                continue
            for j in range(num_q_heads):
                out[b, t, j] = decode_one(query[b, t, j], kv_pool, block_tables[b], visible,
                                          j // group, scale)
    return out
