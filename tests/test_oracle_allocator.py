"""Pins for oracle.block_allocator.

Pins come from the pages ("Paged attention in LLMs": the worked example,
the waste bound, "any free block fits any request", prefix sharing; the quiz
page's table: copy-on-write for beam search) and from invariants any correct
allocator of this kind satisfies.  Brute-force checks recount state from
scratch rather than re-deriving it with the oracle's own formulas.
"""

import json
import os
import random

import pytest

from oracle.block_allocator import BlockAllocator, OutOfBlocks

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")))


def check_invariants(a):
    """Recount the state from the tables and compare with the allocator."""
    counts = [0] * a.num_blocks
    for sid in a.seq_ids():
        for blk in a.block_table(sid):
            counts[blk] += 1
        # a table holds exactly the blocks its length needs
        n = a.seq_len(sid)
        assert len(a.block_table(sid)) * a.block_size >= n
        assert len(a.block_table(sid)) * a.block_size < n + a.block_size or n == 0
    assert counts == a.refcounts()
    free = a.free_list()
    assert len(set(free)) == len(free)
    assert set(free) == {b for b in range(a.num_blocks) if counts[b] == 0}


def fill_per_block(slots, bs):
    fill = {}
    for s in slots:
        fill[s // bs] = fill.get(s // bs, 0) + 1
    return fill


def test_worked_example_through_allocator():
    g = GOLDEN["worked_example"]["paged"]
    a = BlockAllocator(num_blocks=10, block_size=g["block_size"])
    a.add_seq(0)
    slots, cow = a.append(0, GOLDEN["worked_example"]["reply_tokens"])
    table = a.block_table(0)
    assert cow == []
    assert len(table) == g["blocks"]
    assert len(table) * g["block_size"] == g["held"]
    assert len(slots) == g["used"]
    assert len(table) * g["block_size"] - len(slots) == g["wasted"]
    fill = fill_per_block(slots, g["block_size"])
    assert [fill[b] for b in table] == g["fill"]
    check_invariants(a)


def test_default_and_given_pop_order():
    a = BlockAllocator(8, 4)
    a.add_seq(1)
    a.append(1, 9)
    assert a.block_table(1) == [0, 1, 2]
    order = [5, 3, 7, 0, 1, 2, 4, 6]
    b = BlockAllocator(8, 4, initial_order=order)
    b.add_seq(1)
    b.append(1, 9)
    assert b.block_table(1) == [5, 3, 7]
    assert b.free_list() == [0, 1, 2, 4, 6]


def test_slots_are_distinct_and_inside_own_blocks():
    rnd = random.Random(3)
    a = BlockAllocator(200, 7, initial_order=rnd.sample(range(200), 200))
    owner = {}
    for sid in range(12):
        a.add_seq(sid)
    for _ in range(40):
        sid = rnd.randrange(12)
        slots, _ = a.append(sid, rnd.randint(1, 9))
        for s in slots:
            assert s not in owner
            owner[s] = sid
            assert s // 7 in a.block_table(sid)
    # every token of a request got exactly one slot
    for sid in range(12):
        assert sum(1 for o in owner.values() if o == sid) == a.seq_len(sid)
    check_invariants(a)


def test_lifo_reuse():
    a = BlockAllocator(6, 2)
    a.add_seq(0)
    a.append(0, 5)  # blocks 0,1,2
    a.free_seq(0)  # pushed 0,1,2 -> top is 2
    assert a.free_list()[:3] == [2, 1, 0]
    a.add_seq(1)
    a.append(1, 3)
    assert a.block_table(1) == [2, 1]


def test_any_free_block_fits_after_churn():
    """After arbitrary churn a request for k blocks succeeds iff k are free."""
    rnd = random.Random(11)
    bs = 4
    a = BlockAllocator(64, bs, initial_order=rnd.sample(range(64), 64))
    live = []
    for step in range(400):
        if live and rnd.random() < 0.45:
            a.free_seq(live.pop(rnd.randrange(len(live))))
        else:
            sid = 1000 + step
            k = rnd.randint(1, 12)
            a.add_seq(sid)
            if a.num_free() >= k:
                a.append(sid, k * bs)
                assert len(a.block_table(sid)) == k
                live.append(sid)
            else:
                before = (a.free_list(), a.refcounts())
                with pytest.raises(OutOfBlocks):
                    a.append(sid, k * bs)
                assert (a.free_list(), a.refcounts()) == before
                a.free_seq(sid)
        check_invariants(a)


def test_waste_bound_per_request():
    rnd = random.Random(5)
    for bs in (1, 3, 5, 16):
        a = BlockAllocator(4000, bs)
        for sid in range(30):
            a.add_seq(sid)
            n = rnd.randint(1, 300)
            a.append(sid, n)
            held = len(a.block_table(sid)) * bs
            assert 0 <= held - n <= bs - 1


def test_fork_shares_blocks():
    a = BlockAllocator(32, 4)
    a.add_seq(0)
    a.append(0, 10)
    a.fork(0, 1)
    a.fork(0, 2)
    assert a.block_table(1) == a.block_table(0) == a.block_table(2)
    assert all(a.refcount(b) == 3 for b in a.block_table(0))
    check_invariants(a)


def test_copy_on_write_partial_block():
    """k beams sharing a partial block: k-1 copies, the last writes in place."""
    bs = 16
    a = BlockAllocator(64, bs)
    a.add_seq(100)
    a.append(100, 2 * bs + 2)  # 2 full blocks + 2 tokens in the third
    for beam in range(4):
        a.fork(100, beam)
    a.free_seq(100)
    shared = a.block_table(0)
    partial = shared[-1]
    assert a.refcount(partial) == 4
    slots, cow = a.append_batch([0, 1, 2, 3], 1)
    assert [src for src, _ in cow] == [partial] * 3
    dsts = [dst for _, dst in cow]
    assert len(set(dsts)) == 3 and partial not in dsts
    # beams 0..2 now own a copy; beam 3 writes into the original
    for beam in range(3):
        t = a.block_table(beam)
        assert t[:-1] == shared[:-1] and t[-1] == dsts[beam]
        assert slots[beam] == dsts[beam] * bs + 2
    assert a.block_table(3) == shared
    assert slots[3] == partial * bs + 2
    assert a.refcount(partial) == 1
    assert all(a.refcount(b) == 4 for b in shared[:-1])
    check_invariants(a)


def test_full_shared_blocks_are_never_copied():
    a = BlockAllocator(64, 4)
    a.add_seq(0)
    a.append(0, 8)  # exactly two full blocks
    a.fork(0, 1)
    slots, cow = a.append_batch([0, 1], 3)
    assert cow == []
    assert a.block_table(0)[:2] == a.block_table(1)[:2]
    assert a.block_table(0)[2] != a.block_table(1)[2]
    check_invariants(a)


def test_out_of_blocks_is_atomic():
    a = BlockAllocator(5, 4)
    a.add_seq(0)
    a.add_seq(1)
    a.append(0, 9)  # 3 blocks
    snap = (a.free_list(), a.refcounts(), a.block_table(0), a.block_table(1), a.seq_len(0), a.seq_len(1))
    with pytest.raises(OutOfBlocks):
        a.append_batch([1, 0], 8)  # needs 2 + 2 blocks, only 2 free
    assert snap == (a.free_list(), a.refcounts(), a.block_table(0), a.block_table(1), a.seq_len(0), a.seq_len(1))


def test_bad_initial_order():
    with pytest.raises(ValueError):
        BlockAllocator(4, 2, initial_order=[0, 1, 1, 2])
