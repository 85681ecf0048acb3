"""The balanced decode schedule's integer arithmetic, restated on the host.

The decode kernel gives CTA c of C the work units [floor(U c / C),
floor(U (c+1) / C)) of the U = Hkv * sum_b ceil(L_b / bs) units (request b,
KV head h, block k), in that order; a (b, h) whose units span several CTAs
leaves a partial in slot 0 of each CTA whose range starts inside it and in
slot 1 of the CTA whose range it ends; the merge finds the covering CTAs with
"the CTA of unit u" = ceil(C (u + 1) / U) - 1.  These checks run the same
formulas over random batches: every unit is taken exactly once, the covering
CTAs of every (b, h) are exactly the ones the merge visits, and no two
partials land in the same slot.  The GPU tests check the kernels themselves.
"""

import numpy as np


def stream_begin(total, c, ctas):
    return total * c // ctas


def stream_cta_of(total, u, ctas):
    return (ctas * (u + 1) + total - 1) // total - 1


def check_batch(lens, hkv, bs, ctas):
    nblk = [-(-n // bs) for n in lens]
    prefix = np.concatenate([[0], np.cumsum(nblk)]).astype(np.int64)
    total = hkv * int(prefix[-1])
    if total == 0:
        return
    owner = np.full(total, -1)
    slots = {}
    for c in range(ctas):
        lo, hi = stream_begin(total, c, ctas), stream_begin(total, c + 1, ctas)
        assert np.all(owner[lo:hi] == -1)
        owner[lo:hi] = c
        u = lo
        while u < hi:  # the CTA's segments of constant (b, h)
            b = int(np.searchsorted(hkv * prefix, u, side="right")) - 1
            while nblk[b] == 0:
                b -= 1
            nb = nblk[b]
            h = (u - hkv * int(prefix[b])) // nb
            start = hkv * int(prefix[b]) + h * nb
            cnt = min(start + nb, hi) - u
            if not (u == start and cnt == nb):  # a cut segment: one partial slot
                slot = 0 if u == lo else 1
                assert (c, slot) not in slots
                slots[(c, slot)] = (b, h)
            u += cnt
    assert np.all(owner >= 0)
    for b, nb in enumerate(nblk):
        for h in range(hkv if nb else 0):
            us = hkv * int(prefix[b]) + h * nb
            c0, c1 = stream_cta_of(total, us, ctas), stream_cta_of(total, us + nb - 1, ctas)
            assert c0 == owner[us] and c1 == owner[us + nb - 1]
            if c0 == c1:
                continue
            visited = set()
            for c in range(c0, c1 + 1):
                cb = stream_begin(total, c, ctas)
                if stream_begin(total, c + 1, ctas) <= cb:
                    continue  # an empty range: the merge skips it
                visited.add((c, 0 if cb >= us else 1))
            assert visited == {k for k, v in slots.items() if v == (b, h)}


def test_schedule_arithmetic_random_batches():
    rng = np.random.default_rng(354)
    for _ in range(400):
        batch = int(rng.integers(1, 30))
        lens = [int(x) for x in rng.choice([0, 1, 15, 16, 17, int(rng.integers(1, 400))], size=batch)]
        check_batch(lens, int(rng.integers(1, 6)), int(rng.choice([16, 32])), int(rng.choice([1, 3, 7, 64, 296])))


def test_schedule_arithmetic_workload_shapes():
    check_batch([2336] * 64, 8, 16, 296)  # the Llama-3-8B decode shape, uniform lengths
    check_batch([32768] * 4, 8, 16, 296)  # the long-context case: each (b, h) over ~9 CTAs
    check_batch([40000], 2, 16, 296)  # one request cut across every CTA
    check_batch([1, 0, 3], 2, 16, 296)  # fewer units than CTAs


# --------------------------------------------------------------------------
# The tcgen05 consumer's walk: the producer warp cuts each CTA's range into
# segments of constant (b, h) and each segment into tiles of up to
# tile_tokens / bs blocks, the largest multiple of that up to 32 table
# entries at a time; flags mark a segment's first
# and last tile, a segment covering its whole (b, h), and the CTA's final
# tile.  Restated here from the kernel's loop (request advance by lengths,
# skipping empty requests) and checked against the unit arithmetic above.
# --------------------------------------------------------------------------
FIRST, LAST, COMPLETE, FINAL = 1, 2, 4, 8


def tile_walk(lens, hkv, bs, total, lo, hi, tile_tokens=128):
    """Tiles (b, h, first block, blocks, flags, segment) of the range [lo, hi)."""
    nblk = [-(-n // bs) for n in lens]
    prefix = np.concatenate([[0], np.cumsum(nblk)]).astype(np.int64)
    tile_blocks = tile_tokens // bs
    chunk = 32 // tile_blocks * tile_blocks
    b = int(np.searchsorted(hkv * prefix, lo, side="right")) - 1
    while nblk[b] == 0:
        b -= 1
    r = lo - hkv * int(prefix[b])
    h, k = r // nblk[b], r % nblk[b]
    nb = nblk[b]
    u, seg, tiles = lo, 0, []
    while u < hi:
        cnt = min(nb - k, hi - u)
        complete = k == 0 and cnt == nb
        for base in range(0, cnt, chunk):
            n32 = min(chunk, cnt - base)
            for t0 in range(0, n32, tile_blocks):
                n = min(tile_blocks, n32 - t0)
                flags = ((FIRST if base + t0 == 0 else 0) | (LAST if base + t0 + n == cnt else 0)
                         | (COMPLETE if complete else 0) | (FINAL if u + base + t0 + n == hi else 0))
                tiles.append((b, h, k + base + t0, n, flags, seg))
        u += cnt
        seg += 1
        k = 0
        h += 1
        if h == hkv:
            h = 0
            b += 1
            while b < len(lens) and nblk[b] == 0:
                b += 1
            nb = nblk[b] if b < len(lens) else 0
    return tiles


def check_tiles(lens, hkv, bs, ctas, tile_tokens=128):
    nblk = [-(-n // bs) for n in lens]
    prefix = np.concatenate([[0], np.cumsum(nblk)]).astype(np.int64)
    total = hkv * int(prefix[-1])
    if total == 0:
        return
    seen = np.zeros(total, dtype=np.int64)
    for c in range(ctas):
        lo, hi = stream_begin(total, c, ctas), stream_begin(total, c + 1, ctas)
        tiles = tile_walk(lens, hkv, bs, total, lo, hi, tile_tokens)
        if lo == hi:
            assert tiles == []
            continue
        assert tiles[-1][4] & FINAL and all(not (t[4] & FINAL) for t in tiles[:-1])
        for b, h, k0, n, flags, seg in tiles:
            assert 1 <= n <= tile_tokens // bs and k0 + n <= nblk[b]
            u0 = hkv * int(prefix[b]) + h * nblk[b] + k0
            seen[u0:u0 + n] += 1
        # segments: consecutive tiles of one (b, h), FIRST on the first, LAST on the last
        segs = {}
        for t in tiles:
            segs.setdefault(t[5], []).append(t)
        for s, ts in segs.items():
            assert len({(t[0], t[1]) for t in ts}) == 1
            assert ts[0][4] & FIRST and all(not (t[4] & FIRST) for t in ts[1:])
            assert ts[-1][4] & LAST and all(not (t[4] & LAST) for t in ts[:-1])
            b, h = ts[0][0], ts[0][1]
            covered = sum(t[3] for t in ts)
            whole = ts[0][2] == 0 and covered == nblk[b]
            assert all(bool(t[4] & COMPLETE) == whole for t in ts)
            if not whole:
                # a cut (b, h): slot 0 for the CTA's first segment, 1 otherwise --
                # the slot the merge reads for this CTA
                us = hkv * int(prefix[b]) + h * nblk[b]
                assert (0 if lo >= us else 1) == (0 if s == 0 else 1)
    assert np.all(seen == 1)


def test_tile_walk_random_batches():
    rng = np.random.default_rng(355)
    for _ in range(300):
        batch = int(rng.integers(1, 30))
        lens = [int(x) for x in rng.choice([0, 1, 15, 16, 17, 127, 128, 129, int(rng.integers(1, 3000))],
                                           size=batch)]
        check_tiles(lens, int(rng.integers(1, 6)), int(rng.choice([16, 32])), int(rng.choice([1, 3, 7, 64, 148])),
                    int(rng.choice([64, 96, 128])))


def test_tile_walk_workload_shapes():
    check_tiles([2336] * 64, 8, 16, 148)
    check_tiles([32768] * 4, 8, 16, 148)
    check_tiles([40000], 2, 16, 148)
    check_tiles([1, 0, 3], 2, 16, 148)
    check_tiles([0, 0, 5000, 0, 7, 0], 3, 32, 148)


# --------------------------------------------------------------------------
# Overhead-weighted split: each (b, h) with nb > 0 blocks counts as nb + X
# units, the last X of them virtual (no data), so CTAs that cover many short
# (b, h) take fewer real blocks.  A CTA skips segments that hold only virtual
# units (they still count as segments for the partial-slot rule); the merge
# finds the covering CTAs from the (b, h)'s real units only.
# --------------------------------------------------------------------------
def weighted_walk(lens, hkv, bs, ctas, extra, tile_tokens=128):
    nblk = [-(-n // bs) for n in lens]
    units = [nb + extra if nb else 0 for nb in nblk]
    prefix = np.concatenate([[0], np.cumsum(units)]).astype(np.int64)
    total = hkv * int(prefix[-1])
    tile_blocks = tile_tokens // bs
    out = {}
    for c in range(ctas):
        lo, hi = stream_begin(total, c, ctas), stream_begin(total, c + 1, ctas)
        segs, u, seg = [], lo, 0
        if lo < hi:
            b = int(np.searchsorted(hkv * prefix, lo, side="right")) - 1
            while units[b] == 0:
                b -= 1
            r = lo - hkv * int(prefix[b])
            h, k = r // units[b], r % units[b]
            while u < hi:
                nbu, nb = units[b], nblk[b]
                cnt = min(nbu - k, hi - u)
                real = max(0, min(k + cnt, nb) - k)
                if real:
                    segs.append((b, h, k, real, k == 0 and real == nb, seg,
                                 -(-real // tile_blocks)))
                u += cnt
                seg += 1
                k = 0
                h += 1
                if h == hkv:
                    h = 0
                    b += 1
                    while b < len(lens) and units[b] == 0:
                        b += 1
        out[c] = (lo, hi, segs)
    return nblk, units, prefix, total, out


def check_weighted(lens, hkv, bs, ctas, extra):
    nblk, units, prefix, total, out = weighted_walk(lens, hkv, bs, ctas, extra)
    if total == 0:
        return
    seen = {}
    slots = {}
    for c, (lo, hi, segs) in out.items():
        for b, h, k, real, complete, seg, _ in segs:
            for blk in range(k, k + real):
                assert (b, h, blk) not in seen
                seen[(b, h, blk)] = c
            if not complete:
                slot = 0 if seg == 0 else 1
                assert (c, slot) not in slots
                slots[(c, slot)] = (b, h)
    assert len(seen) == hkv * sum(nblk)  # every real block exactly once
    for b, nb in enumerate(nblk):
        for h in range(hkv if nb else 0):
            us = hkv * int(prefix[b]) + h * units[b]
            c0, c1 = stream_cta_of(total, us, ctas), stream_cta_of(total, us + nb - 1, ctas)
            assert c0 == seen[(b, h, 0)] and c1 == seen[(b, h, nb - 1)]
            if c0 == c1:
                continue
            visited = set()
            for c in range(c0, c1 + 1):
                cb = stream_begin(total, c, ctas)
                if stream_begin(total, c + 1, ctas) <= cb:
                    continue
                visited.add((c, 0 if cb >= us else 1))
            assert visited == {kk for kk, v in slots.items() if v == (b, h)}


def test_weighted_split_random_batches():
    rng = np.random.default_rng(356)
    for _ in range(300):
        batch = int(rng.integers(1, 30))
        lens = [int(x) for x in rng.choice([0, 1, 15, 16, 17, 127, 128, 129, int(rng.integers(1, 3000))],
                                           size=batch)]
        check_weighted(lens, int(rng.integers(1, 6)), int(rng.choice([16, 32])),
                       int(rng.choice([1, 3, 7, 64, 148])), int(rng.choice([0, 1, 5, 12, 40])))


def test_weighted_split_evens_out_segments():
    """At the Llama-3-8B lengths the weighting narrows the spread of real
    blocks + per-segment cost over the 148 CTAs."""
    import workloads

    lens = [int(x) for x in workloads.plan("llama8b").seq_lens]

    def spread(extra, cost=12):
        _, _, _, _, out = weighted_walk(lens, 8, 16, 148, extra)
        work = [sum(s[3] + cost for s in segs) for _, _, segs in out.values()]
        return max(work) - min(work)

    assert spread(12) < spread(0) / 2
