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
