"""Pins for oracle.paged_attention.decode / gather_kv.

The quiz page's sketch ("Conceptual: PagedAttention block lookup") defines
decode as "gather K/V through the block table, then standard scaled dot
product attention".  These pins tie the oracle to things other than itself:

* the pool is built from contiguous K/V with numpy reshape/transpose and a
  block-level placement (no per-position block/offset arithmetic), so the
  gather must reproduce the contiguous K/V ("the sequence stays in order",
  "Paged attention in LLMs", section "Keeping track: the block table");
* torch's scaled_dot_product_attention in float64 on CPU (a library routine)
  on the contiguous K/V, with query-head groups expanded by
  repeat_interleave;
* closed forms: length 1 returns V[0]; scale 0 returns the mean of V; two
  positions give logistic weights; constant V per KV head reveals the
  query-head -> KV-head mapping;
* invariance under any permutation of the physical blocks;
* the contiguous-reservation decode equals the paged decode on the same
  sequences (and torch SDPA);
* mutation tests: plausible single mistakes planted in a copy of the oracle
  (on the CPU) must each fail at least one pin.
"""

import math

import numpy as np
import pytest
import torch

import oracle.paged_attention as pa


def place_requests(contig_k, contig_v, block_size, num_blocks, rng, fill=np.nan):
    """Pool + block tables holding the given contiguous K/V (library ops only)."""
    hkv, d = contig_k[0].shape[1:]
    pool = np.full((num_blocks, 2, hkv, block_size, d), fill, dtype=np.float64)
    perm = rng.permutation(num_blocks)
    tables, used = [], 0
    for k, v in zip(contig_k, contig_v):
        n = k.shape[0]
        nblk = -(-n // block_size)
        ids = perm[used : used + nblk]
        used += nblk
        for c, x in ((0, k), (1, v)):
            padded = np.full((nblk * block_size, hkv, d), fill)
            padded[:n] = x
            pool[ids, c] = padded.reshape(nblk, block_size, hkv, d).transpose(0, 2, 1, 3)
        tables.append(ids)
    width = max(1, max(len(t) for t in tables))
    table = np.zeros((len(tables), width), dtype=np.int64)
    for i, t in enumerate(tables):
        table[i, : len(t)] = t
    return pool, table


def sdpa_reference(q, k, v, scale):
    """torch SDPA (float64, CPU) for one request: q [Hq,D], k/v [L,Hkv,D]."""
    hq, hkv = q.shape[0], k.shape[1]
    g = hq // hkv
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(g, dim=0)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(g, dim=0)[None]
    qt = torch.from_numpy(q)[None, :, None, :]
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return out[0, :, 0, :].numpy()


def random_case(rng, lens, hq, hkv, d, bs, extra_blocks=5):
    ks = [rng.standard_normal((n, hkv, d)) for n in lens]
    vs = [rng.standard_normal((n, hkv, d)) for n in lens]
    q = rng.standard_normal((len(lens), hq, d))
    nb = sum(-(-n // bs) for n in lens) + extra_blocks
    pool, table = place_requests(ks, vs, bs, nb, rng)
    return q, ks, vs, pool, table


# --------------------------------------------------------------------------
# the pins, written against a module so the mutation test can reuse them
# --------------------------------------------------------------------------
def pin_gather_is_contiguous(m):
    rng = np.random.default_rng(1)
    for bs in (1, 5, 16):
        lens = [1, bs, bs + 1, 3 * bs - 1, 40]
        q, ks, vs, pool, table = random_case(rng, lens, 4, 2, 8, bs)
        for i, n in enumerate(lens):
            k, v = m.gather_kv(pool, table[i], n)
            assert k.shape == (n, 2, 8)
            assert np.array_equal(k, ks[i]) and np.array_equal(v, vs[i])


def pin_sdpa(m):
    rng = np.random.default_rng(2)
    for bs, hq, hkv, d in ((16, 4, 4, 64), (5, 8, 2, 16), (16, 8, 1, 32), (1, 6, 3, 8)):
        lens = [1, 7, bs, 2 * bs + 3, 37]
        q, ks, vs, pool, table = random_case(rng, lens, hq, hkv, d, bs)
        scale = 1.0 / math.sqrt(d)
        got = m.decode(q, pool, table, np.array(lens), scale)
        for i in range(len(lens)):
            ref = sdpa_reference(q[i], ks[i], vs[i], scale)
            np.testing.assert_allclose(got[i], ref, rtol=0, atol=1e-12)


def pin_length_one(m):
    rng = np.random.default_rng(3)
    q, ks, vs, pool, table = random_case(rng, [1, 1], 4, 2, 16, 16)
    got = m.decode(q, pool, table, np.array([1, 1]), 0.7)
    for i in range(2):
        for j in range(4):
            assert np.array_equal(got[i, j], vs[i][0, j // 2])


def pin_scale_zero_is_mean(m):
    rng = np.random.default_rng(4)
    lens = [3, 17, 40]
    q, ks, vs, pool, table = random_case(rng, lens, 2, 2, 8, 16)
    got = m.decode(q, pool, table, np.array(lens), 0.0)
    for i, n in enumerate(lens):
        np.testing.assert_allclose(got[i], vs[i].mean(axis=0), rtol=0, atol=1e-13)


def pin_two_positions_logistic(m):
    """Two keys with dot products a and b: weights 1/(1+e^(s(b-a))) and the rest."""
    d = 4
    q = np.zeros((1, 1, d))
    q[0, 0, 0] = 1.0
    k = np.zeros((2, 1, d))
    k[0, 0, 0], k[1, 0, 0] = 2.0, -1.0  # a = 2, b = -1
    v = np.zeros((2, 1, d))
    v[0, 0] = [1.0, 0.0, 3.0, 0.0]
    v[1, 0] = [0.0, 1.0, 0.0, -2.0]
    pool, table = place_requests([k], [v], 1, 6, np.random.default_rng(5))
    s = 0.5
    w0 = 1.0 / (1.0 + math.exp(s * (-1.0 - 2.0)))
    expect = w0 * v[0, 0] + (1.0 - w0) * v[1, 0]
    got = m.decode(q, pool, table, np.array([2]), s)
    np.testing.assert_allclose(got[0, 0], expect, rtol=0, atol=1e-15)


def pin_head_grouping(m):
    """Constant V per KV head: query head j must read KV head j // g."""
    hkv, g, d, n = 3, 2, 4, 9
    k = np.random.default_rng(6).standard_normal((n, hkv, d))
    v = np.zeros((n, hkv, d))
    for h in range(hkv):
        v[:, h, :] = 10.0 * (h + 1)
    pool, table = place_requests([k], [v], 4, 8, np.random.default_rng(7))
    q = np.random.default_rng(8).standard_normal((1, hkv * g, d))
    got = m.decode(q, pool, table, np.array([n]), 0.3)
    for j in range(hkv * g):
        np.testing.assert_allclose(got[0, j], 10.0 * (j // g + 1), rtol=0, atol=1e-12)


def pin_block_permutation_invariance(m):
    rng = np.random.default_rng(9)
    lens = [33, 50]
    ks = [rng.standard_normal((n, 2, 8)) for n in lens]
    vs = [rng.standard_normal((n, 2, 8)) for n in lens]
    q = rng.standard_normal((2, 4, 8))
    outs = []
    for trial in range(3):
        pool, table = place_requests(ks, vs, 8, 20, np.random.default_rng(100 + trial))
        outs.append(m.decode(q, pool, table, np.array(lens), 0.35))
    for o in outs[1:]:
        np.testing.assert_allclose(o, outs[0], rtol=0, atol=1e-13)


def pin_empty_request(m):
    rng = np.random.default_rng(10)
    q, ks, vs, pool, table = random_case(rng, [5, 5], 2, 1, 8, 4)
    got = m.decode(q, pool, table, np.array([0, 5]), 0.5)
    assert np.array_equal(got[0], np.zeros((2, 8)))
    assert np.isfinite(got[1]).all()


def pin_decode_one(m):
    rng = np.random.default_rng(11)
    lens = [9, 21]
    q, ks, vs, pool, table = random_case(rng, lens, 4, 2, 8, 4)
    full = m.decode(q, pool, table, np.array(lens), 0.4)
    for i in range(2):
        for j in range(4):
            one = m.decode_one(q[i, j], pool, table[i], lens[i], j // 2, 0.4)
            np.testing.assert_allclose(one, full[i, j], rtol=0, atol=1e-14)


def pin_multi_reduces_to_decode(m):
    """T = 1 is exactly the single-token decode; token t of T equals a
    single-token decode over the first L - T + t + 1 positions."""
    rng = np.random.default_rng(12)
    lens = [9, 21, 3]
    q, ks, vs, pool, table = random_case(rng, lens, 4, 2, 8, 4)
    one = m.decode_multi(q[:, None], pool, table, np.array(lens), 0.4)
    np.testing.assert_array_equal(one[:, 0], m.decode(q, pool, table, np.array(lens), 0.4))
    T = 4
    qm = rng.standard_normal((3, T, 4, 8))
    got = m.decode_multi(qm, pool, table, np.array(lens), 0.4)
    for b, n in enumerate(lens):
        for t in range(T):
            vis = n - T + t + 1
            want = m.decode(qm[b:b + 1, t], pool, table[b:b + 1], np.array([max(vis, 0)]), 0.4)
            np.testing.assert_array_equal(got[b, t], want[0])


def pin_multi_causal_sdpa(m):
    """Against torch SDPA (fp64) with an explicit causal mask on contiguous K/V."""
    rng = np.random.default_rng(13)
    lens, T, hq, hkv, d = [7, 30, 16], 5, 8, 2, 16
    ks = [rng.standard_normal((n, hkv, d)) for n in lens]
    vs = [rng.standard_normal((n, hkv, d)) for n in lens]
    pool, table = place_requests(ks, vs, 4, 20, rng)
    q = rng.standard_normal((len(lens), T, hq, d))
    got = m.decode_multi(q, pool, table, np.array(lens), 0.3)
    for b, n in enumerate(lens):
        g = hq // hkv
        kt = torch.from_numpy(ks[b]).permute(1, 0, 2).repeat_interleave(g, dim=0)[None]
        vt = torch.from_numpy(vs[b]).permute(1, 0, 2).repeat_interleave(g, dim=0)[None]
        qt = torch.from_numpy(q[b]).permute(1, 0, 2)[None]  # [1, Hq, T, D]
        pos = torch.arange(n)[None, :]
        qpos = (n - T + torch.arange(T))[:, None]
        mask = pos <= qpos  # [T, n]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.3)
        ref = ref[0].permute(1, 0, 2).numpy()
        np.testing.assert_allclose(got[b], ref, rtol=0, atol=1e-12)


def pin_multi_short_request(m):
    """Query tokens before the request's start attend to nothing: output 0."""
    rng = np.random.default_rng(14)
    q, ks, vs, pool, table = random_case(rng, [2], 2, 1, 8, 4)
    qm = rng.standard_normal((1, 4, 2, 8))
    got = m.decode_multi(qm, pool, table, np.array([2]), 0.5)
    assert np.array_equal(got[0, :2], np.zeros((2, 2, 8)))
    np.testing.assert_allclose(got[0, 3], m.decode(qm[:, 3], pool, table, np.array([2]), 0.5)[0], atol=0)


def contiguous_cache(ks, vs, max_len, fill=np.nan):
    """[B, 2, Hkv, max_len, D] reservation per request (library ops only);
    positions past each request's length hold ``fill``."""
    hkv, d = ks[0].shape[1:]
    cache = np.full((len(ks), 2, hkv, max_len, d), fill)
    for b, (k, v) in enumerate(zip(ks, vs)):
        cache[b, 0, :, :k.shape[0]] = k.transpose(1, 0, 2)
        cache[b, 1, :, :v.shape[0]] = v.transpose(1, 0, 2)
    return cache


def pin_contiguous_matches_paged(m):
    """The contiguous reservation and the paged pool hold the same sequence,
    so decode over either gives the same output (the reservation's unused
    tail, NaN here, is never read)."""
    rng = np.random.default_rng(15)
    lens = [1, 17, 40, 0, 33]
    q, ks, vs, pool, table = random_case(rng, lens, 8, 2, 16, 4)
    cache = contiguous_cache(ks, vs, 48)
    got = m.decode_contiguous(q, cache, np.array(lens), 0.3)
    want = m.decode(q, pool, table, np.array(lens), 0.3)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    assert np.array_equal(got[3], np.zeros((8, 16)))


def pin_contiguous_sdpa(m):
    """Against torch SDPA (fp64) on the request's keys and values."""
    rng = np.random.default_rng(16)
    lens, hq, hkv, d = [5, 64, 23], 12, 3, 32
    ks = [rng.standard_normal((n, hkv, d)) for n in lens]
    vs = [rng.standard_normal((n, hkv, d)) for n in lens]
    q = rng.standard_normal((len(lens), hq, d))
    got = m.decode_contiguous(q, contiguous_cache(ks, vs, 64), np.array(lens), 0.2)
    for b in range(len(lens)):
        np.testing.assert_allclose(got[b], sdpa_reference(q[b], ks[b], vs[b], 0.2), rtol=0, atol=1e-12)


DECODE_PINS = [
    pin_gather_is_contiguous,
    pin_sdpa,
    pin_length_one,
    pin_scale_zero_is_mean,
    pin_two_positions_logistic,
    pin_head_grouping,
    pin_block_permutation_invariance,
    pin_empty_request,
    pin_decode_one,
    pin_multi_reduces_to_decode,
    pin_multi_causal_sdpa,
    pin_multi_short_request,
    pin_contiguous_matches_paged,
    pin_contiguous_sdpa,
]


@pytest.mark.parametrize("pin", DECODE_PINS, ids=lambda f: f.__name__)
def test_decode_pin(pin):
    pin(pa)


# --------------------------------------------------------------------------
# mutation test: each planted mistake must break at least one pin
# --------------------------------------------------------------------------
MUTATIONS = {
    "gqa_modulo": ("h = j // group", "h = j % num_kv_heads"),
    "block_index_swapped": ("[pos // block_size]", "[pos % block_size]"),
    "offset_swapped": ("offset = pos % block_size", "offset = pos // block_size"),
    "scale_dropped": ("logits = scale * (keys", "logits = (keys"),
    "sign_flipped": ("weights = np.exp(logits - logits.max())\n            weights /= weights.sum()",
                     "weights = np.exp(logits.max() - logits)\n            weights /= weights.sum()"),
    "k_v_swapped": ("keys = kv_pool[phys, 0, :, offset, :]", "keys = kv_pool[phys, 1, :, offset, :]"),
    "not_normalised": ("            weights /= weights.sum()\n            out[b, j]", "            out[b, j]"),
    "keys_for_values": ("out[b, j] = weights @ values[:, h, :]", "out[b, j] = weights @ keys[:, h, :]"),
    "off_by_one_length": ("pos = np.arange(seq_len)", "pos = np.arange(1, seq_len + 1)"),
    "multi_not_causal": ("visible = int(seq_lens[b]) - tokens + t + 1", "visible = int(seq_lens[b])"),
    "contiguous_k_v_swapped": ("keys = kv_cache[b, 0, j // group", "keys = kv_cache[b, 1, j // group"),
    "contiguous_reads_past_length": ("keys = kv_cache[b, 0, j // group, :seq_len]",
                                     "keys = kv_cache[b, 0, j // group, :seq_len + 1]"),
    "contiguous_gqa_modulo": ("values = kv_cache[b, 1, j // group, :seq_len]",
                              "values = kv_cache[b, 1, j % num_kv_heads, :seq_len]"),
    "multi_off_by_one": ("visible = int(seq_lens[b]) - tokens + t + 1", "visible = int(seq_lens[b]) - tokens + t"),
}


def mutated_module(old, new):
    import types

    src = open(pa.__file__).read()
    assert src.count(old) >= 1, old
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name):
    mod = mutated_module(*MUTATIONS[name])
    failed = []
    for pin in DECODE_PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mod)
        except Exception:  # assertion or indexing error: the pin caught it
            failed.append(pin.__name__)
    assert failed, f"mutation {name} passed every pin"
