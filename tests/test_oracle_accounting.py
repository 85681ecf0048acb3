"""Pins for oracle.accounting against the numbers the pages print.

Golden values: tests/golden/worked_example.json, from "Paged attention in
LLMs", sections "A worked example" and "Why the memory gets wasted".
"""

import json
import os

import pytest

from oracle import accounting

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")))


def test_worked_example_contiguous():
    g = GOLDEN["worked_example"]
    held, used, wasted = accounting.contiguous(32, g["reply_tokens"])
    assert (held, used, wasted) == (
        g["contiguous_reservation"]["held"],
        g["contiguous_reservation"]["used"],
        g["contiguous_reservation"]["wasted"],
    )


def test_worked_example_paged():
    g = GOLDEN["worked_example"]
    p = g["paged"]
    blocks, held, used, wasted = accounting.paged(g["reply_tokens"], p["block_size"])
    assert (blocks, held, used, wasted) == (p["blocks"], p["held"], p["used"], p["wasted"])
    assert accounting.block_fill(g["reply_tokens"], p["block_size"]) == p["fill"]


def test_reservation_example():
    g = GOLDEN["reservation_example"]
    assert accounting.contiguous(g["reserved"], g["used"])[2] == g["idle"]


def test_gap_example():
    g = GOLDEN["gap_example"]
    assert sum(g["gaps"]) == g["free_total"]
    assert accounting.contiguous_fits(g["gaps"], g["request"]) is g["contiguous_fits"]
    # the same free slots, cut into blocks of 2, do host the request
    assert accounting.paged_fits(g["free_total"] // 2, g["request"], 2)


def test_waste_bound_brute_force():
    """Waste per request is below one block ("Why this helps so much").

    Brute force: the held size is the smallest multiple of block_size that
    is not below the length, found by counting up.
    """
    bound = GOLDEN["waste_bound_example"]
    assert max(accounting.paged(n, bound["block_size"])[3] for n in range(1, 200)) == bound[
        "max_waste_per_request"
    ]
    for bs in range(1, 21):
        for n in range(0, 130):
            held = 0
            while held < n:
                held += bs
            blocks, h, used, wasted = accounting.paged(n, bs)
            assert h == held and blocks * bs == held and used == n
            assert 0 <= wasted <= bs - 1
            assert sum(accounting.block_fill(n, bs)) == n
            assert len(accounting.block_fill(n, bs)) == blocks


def test_contiguous_rejects_overflow():
    with pytest.raises(ValueError):
        accounting.contiguous(10, 11)


def test_allocator_stats_worked_example_and_sharing():
    from oracle.block_allocator import BlockAllocator

    g = GOLDEN["worked_example"]
    a = BlockAllocator(10, g["paged"]["block_size"])
    a.add_seq(0)
    a.append(0, g["reply_tokens"])
    st = accounting.allocator_stats(a)
    assert st["tokens"] == g["paged"]["used"]
    assert st["logical_slots"] == g["paged"]["held"]
    assert st["logical_slots"] - st["tokens"] == g["paged"]["wasted"]
    assert st["physical_blocks"] == g["paged"]["blocks"] and st["free_blocks"] == 10 - 3
    # three forks share every block: logical slots x4, physical unchanged
    for child in (1, 2, 3):
        a.fork(0, child)
    st = accounting.allocator_stats(a)
    assert st["logical_slots"] == 4 * g["paged"]["held"]
    assert st["physical_blocks"] == g["paged"]["blocks"] and st["live_requests"] == 4
