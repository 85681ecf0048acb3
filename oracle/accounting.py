"""Slot accounting of contiguous vs paged KV storage -- test infrastructure only.

"Paged attention in LLMs":

* section "Why the memory gets wasted": a contiguous layout reserves the
  maximum reply length up front; the unused tail of the reservation is
  waste, and free gaps between reservations cannot host a request that needs
  one longer run.
* section "A worked example": the table of slots held / used / wasted for
  one contiguous reservation and for the same reply paged into blocks.
* section "Why this helps so much": paged waste is what is left in the last
  block, at most ``block_size - 1`` slots per request, and any free block
  fits any request.

Definitions used (the page's own): held = slots reserved for the request,
used = tokens stored, wasted = held - used.
"""


def contiguous(reserved_slots, used_tokens):
    """One contiguous reservation: (held, used, wasted)."""
    if used_tokens > reserved_slots:
        raise ValueError("reply longer than the reservation")
    return reserved_slots, used_tokens, reserved_slots - used_tokens


def paged(used_tokens, block_size):
    """Paged into fixed-size blocks: (blocks, held, used, wasted)."""
    blocks = -(-used_tokens // block_size)  # ceiling division
    held = blocks * block_size
    return blocks, held, used_tokens, held - used_tokens


def block_fill(used_tokens, block_size):
    """Tokens stored in each block of a request, in table order."""
    fill = []
    left = used_tokens
    while left > 0:
        fill.append(min(block_size, left))
        left -= block_size
    return fill


def contiguous_fits(free_gaps, request_slots):
    """A contiguous request needs one gap at least as long as itself."""
    return any(gap >= request_slots for gap in free_gaps)


def paged_fits(num_free_blocks, request_slots, block_size):
    """Any free block fits any request: only the block count matters."""
    return num_free_blocks * block_size >= request_slots


def allocator_stats(alloc):
    """Occupancy of a block allocator model, counted from its tables.

    tokens          -- sum of the live requests' lengths
    logical_slots   -- sum over requests of (blocks in its table) * block_size
    physical_blocks -- distinct physical blocks referenced by any table
    live_requests   -- number of requests
    free_blocks     -- blocks on the free list
    Internal waste is logical_slots - tokens ("Why this helps so much": the
    tail of each request's last block); sharing saves logical_slots -
    physical_blocks * block_size ("Sharing blocks").
    """
    ids = alloc.seq_ids()
    tables = [alloc.block_table(s) for s in ids]
    return {
        "tokens": sum(alloc.seq_len(s) for s in ids),
        "logical_slots": sum(len(t) for t in tables) * alloc.block_size,
        "physical_blocks": len({b for t in tables for b in t}),
        "live_requests": len(ids),
        "free_blocks": alloc.num_free(),
    }
