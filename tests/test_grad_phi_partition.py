"""The split of grad_phi's work over persistent CTAs at n = 8 and n = 16 (host
arithmetic only; no GPU).

grad_phi = sum over tokens of x_t u_t^T is cut into units (phi block, 128-token
tile), numbered block-major: unit u = blk * ntt + tile.  CTA b of G takes the
contiguous units [b U / G, (b + 1) U / G) (integer division), so the owner of
unit u is ((u + 1) G - 1) / U.  Inside its range a CTA walks its blocks in
order: a block it covers whole is written straight to grad_phi; a block it
covers in part goes to one of its two partial slots, slot 0 for the first
block of its range and slot 1 for the last.  The finish kernel then adds, for
every block touched by more than one CTA, the slots of the CTAs from the first
owner to the last, taking slot 0 of a CTA whose range starts inside that block
and slot 1 otherwise.

These tests restate that scheme and check, over many sizes and grids, that it
is a partition: every unit belongs to exactly one CTA; a CTA never needs a
third slot; a block touched by one CTA is written whole by it; and the slots
the finisher reads for a block are exactly the ones its writers wrote, with no
slot written twice.
"""
import itertools

import pytest


def writers(nblk, ntt, G):
    """What each CTA writes: {(b, slot): blk} for partial slots and the set of
    blocks written whole, following the kernels' walk over a CTA's range."""
    U = nblk * ntt
    slots, whole, covered = {}, [], []
    for b in range(G):
        lo, hi = b * U // G, (b + 1) * U // G
        covered.extend(range(lo, hi))
        b0 = lo // ntt
        b1 = (hi - 1) // ntt if hi > lo else b0 - 1
        for blk in range(b0, b1 + 1):
            si = blk - b0
            s_lo, s_hi = max(blk * ntt, lo), min((blk + 1) * ntt, hi)
            if s_lo == blk * ntt and s_hi == (blk + 1) * ntt:
                whole.append(blk)
            else:
                key = (b, 0 if si == 0 else 1)
                assert key not in slots, f"CTA {b} writes slot {key[1]} twice"
                slots[key] = blk
    return slots, whole, covered


def finisher(nblk, ntt, G):
    """What the finish kernel reads: {blk: [(b, slot), ...]} for the blocks that
    more than one CTA touched."""
    U = nblk * ntt

    def owner(u):
        return ((u + 1) * G - 1) // U

    reads = {}
    for blk in range(nblk):
        bfirst, blast = owner(blk * ntt), owner((blk + 1) * ntt - 1)
        if bfirst == blast:
            continue
        reads[blk] = [(b, 0 if (b * U // G) // ntt == blk else 1)
                      for b in range(bfirst, blast + 1)]
    return reads


def _cases():
    # blocks: n = 8 at C = 136 is 8 x 2 blocks of 128 channels, n = 16 at C = 7168
    # is 16 x 56; tiles: T / 128 rounded up; grids up to the kernels' 256
    for nblk, ntt in itertools.product((1, 2, 3, 16, 17, 112, 896), (1, 2, 3, 8, 33, 128)):
        U = nblk * ntt
        for G in sorted({1, 2, 3, 7, min(U, 148), min(U, 256), min(U, 255), U if U <= 256 else 1}):
            if 1 <= G <= min(U, 256):
                yield nblk, ntt, G


CASES = list(_cases())


@pytest.mark.parametrize("nblk,ntt,G", CASES)
def test_units_split_into_a_partition(nblk, ntt, G):
    slots, whole, covered = writers(nblk, ntt, G)
    U = nblk * ntt
    assert sorted(covered) == list(range(U))      # every unit exactly once
    owner = lambda u: ((u + 1) * G - 1) // U
    for b in range(G):                             # the closed-form owner agrees
        for u in range(b * U // G, (b + 1) * U // G):
            assert owner(u) == b
    reads = finisher(nblk, ntt, G)
    # a block is either written whole by one CTA or assembled from slots
    assert set(whole).isdisjoint(reads)
    assert len(whole) == len(set(whole))
    assert set(whole) | set(reads) == set(range(nblk))
    # the finisher reads exactly the slots the writers filled, block by block
    written = {}
    for key, blk in slots.items():
        written.setdefault(blk, []).append(key)
    assert {blk: sorted(v) for blk, v in written.items()} == \
        {blk: sorted(v) for blk, v in reads.items()}


def test_cases_cover_blocks_spanning_many_ctas():
    """Among the cases are blocks split over three or more CTAs (a middle CTA
    holding part of one block only) and CTAs whose range spans three or more
    blocks (whole blocks between two partial ones)."""
    many_ctas = many_blocks = False
    for nblk, ntt, G in CASES:
        for reads in finisher(nblk, ntt, G).values():
            many_ctas |= len(reads) >= 3
        U = nblk * ntt
        for b in range(G):
            lo, hi = b * U // G, (b + 1) * U // G
            many_blocks |= (hi - 1) // ntt - lo // ntt >= 2
    assert many_ctas and many_blocks
