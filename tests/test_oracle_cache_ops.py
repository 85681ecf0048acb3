"""Pins for oracle.paged_attention.reshape_and_cache / copy_blocks.

reshape_and_cache is checked against numpy's own multi-index flattening
(``np.ravel_multi_index`` over the pool's shape) with a flat assignment, a
library route that shares no block/offset arithmetic with the oracle, on a
pool pre-filled with a sentinel so stray writes show.  copy_blocks is checked
against whole-array equality and its in-order semantics.  Mutation tests
plant single mistakes in a copy of the oracle (CPU only).
"""

import types

import numpy as np
import pytest

import oracle.paged_attention as pa

SENTINEL = -7.25


def pin_reshape_matches_flat_index(m):
    rng = np.random.default_rng(20)
    for nb, hkv, bs, d in ((6, 2, 4, 8), (9, 3, 5, 4), (8, 1, 1, 2)):
        pool = np.full((nb, 2, hkv, bs, d), SENTINEL)
        t = 7
        slots = rng.choice(nb * bs, size=t, replace=False)
        slots[2] = -1  # padding token
        k = rng.standard_normal((t, hkv, d))
        v = rng.standard_normal((t, hkv, d))
        got = m.reshape_and_cache(pool.copy(), k, v, slots)
        # expected: flat row view [nb*2*hkv*bs, d], rows from ravel_multi_index
        flat = np.full((nb * 2 * hkv * bs, d), SENTINEL)
        for i in range(t):
            if slots[i] < 0:
                continue
            blk, off = np.unravel_index(slots[i], (nb, bs))
            for c, src in ((0, k), (1, v)):
                for h in range(hkv):
                    row = np.ravel_multi_index((blk, c, h, off), (nb, 2, hkv, bs))
                    flat[row] = src[i, h]
        assert np.array_equal(got.reshape(-1, d), flat)


def pin_reshape_last_write_wins(m):
    pool = np.zeros((2, 2, 1, 2, 3))
    k = np.arange(9, dtype=float).reshape(3, 1, 3)
    v = -k
    got = m.reshape_and_cache(pool, k, v, np.array([1, 1, 2]))
    assert np.array_equal(got[0, 0, 0, 1], k[1, 0])
    assert np.array_equal(got[0, 1, 0, 1], v[1, 0])
    assert np.array_equal(got[1, 0, 0, 0], k[2, 0])


def pin_copy_blocks(m):
    rng = np.random.default_rng(21)
    pool = rng.standard_normal((8, 2, 3, 4, 5))
    before = pool.copy()
    got = m.copy_blocks(pool, [(1, 6), (3, 7)])
    assert np.array_equal(got[6], before[1]) and np.array_equal(got[7], before[3])
    for b in (0, 1, 2, 3, 4, 5):
        assert np.array_equal(got[b], before[b])


def pin_copy_blocks_in_order(m):
    pool = np.arange(4 * 2 * 1 * 1 * 2, dtype=float).reshape(4, 2, 1, 1, 2)
    before = pool.copy()
    got = m.copy_blocks(pool, [(0, 1), (1, 2)])
    assert np.array_equal(got[2], before[0])  # second pair sees the first one's result


CACHE_PINS = [pin_reshape_matches_flat_index, pin_reshape_last_write_wins, pin_copy_blocks,
              pin_copy_blocks_in_order]


@pytest.mark.parametrize("pin", CACHE_PINS, ids=lambda f: f.__name__)
def test_cache_pin(pin):
    pin(pa)


MUTATIONS = {
    "k_into_v": ("kv_pool[block, 0, :, offset, :] = key[t]", "kv_pool[block, 1, :, offset, :] = key[t]"),
    "block_offset_swapped": ("block, offset = slot // block_size, slot % block_size",
                             "offset, block = slot // block_size, slot % block_size"),
    "skip_slot_zero": ("if slot < 0:", "if slot <= 0:"),
    "copy_reversed": ("kv_pool[int(dst)] = kv_pool[int(src)].copy()", "kv_pool[int(src)] = kv_pool[int(dst)].copy()"),
    "copy_keys_only": ("kv_pool[int(dst)] = kv_pool[int(src)].copy()", "kv_pool[int(dst), 0] = kv_pool[int(src), 0]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name):
    old, new = MUTATIONS[name]
    src = open(pa.__file__).read()
    assert old in src
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    failed = []
    for pin in CACHE_PINS:
        try:
            pin(mod)
        except Exception:
            failed.append(pin.__name__)
    assert failed, f"mutation {name} passed every pin"
