"""The persistent attention kernel's work split, restated and checked on the CPU.

The kernel runs U units (rollout, head, query-tile pair), unit u with nt(u) KV
iterations, on G CTAs.  The first floor(U / G) waves run whole units; the
iterations of the remaining units, laid end to end from iteration sk0, are cut
into G ranges: CTA c starts at

    begin(c) = sk0 + floor(c * I2 / G)          (I2 iterations in the split part)

and the CTA whose range holds iteration x is

    owner(x) = floor(((x - sk0 + 1) * G - 1) / I2).

A split unit's partial results are merged by the CTAs from owner(first) to
owner(last) of its iterations; the kernel counts its pieces from these two
formulas.  These tests check, over every G up to the kernel's 148 CTAs, that
the ranges partition the split iterations, that owner() inverts begin() onto a
non-empty range, that a unit's pieces are exactly the non-empty ranges between
its owners, and that with iterations * G < 2^31 (the host's bound before a
launch) no intermediate leaves 32 bits.
"""
import random

import pytest

INT32_MAX = 2 ** 31 - 1


def begin(c, sk0, I2, G):
    assert c * I2 <= INT32_MAX
    return sk0 + c * I2 // G


def owner(x, sk0, I2, G):
    assert (x - sk0 + 1) * G <= INT32_MAX
    return ((x - sk0 + 1) * G - 1) // I2


def _check_split(sk0, I2, G):
    ranges = [(begin(c, sk0, I2, G), begin(c + 1, sk0, I2, G)) for c in range(G)]
    # contiguous, ordered, covering [sk0, sk0 + I2)
    assert ranges[0][0] == sk0 and ranges[-1][1] == sk0 + I2
    for (a0, a1), (b0, _) in zip(ranges, ranges[1:]):
        assert a0 <= a1 == b0
    # sizes differ by at most one (an even split)
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1
    # owner() is the inverse of begin(), onto a non-empty range
    for x in range(sk0, sk0 + I2):
        c = owner(x, sk0, I2, G)
        assert 0 <= c < G
        lo, hi = ranges[c]
        assert lo <= x < hi


@pytest.mark.parametrize("G", list(range(1, 149)))
def test_ranges_partition_and_owner_inverts_begin(G):
    rng = random.Random(G)
    cases = [1, 2, G - 1, G, G + 1, 2 * G - 1, 3 * G + 7] + [rng.randint(1, 900) for _ in range(6)]
    for I2 in cases:
        if I2 < 1:
            continue
        _check_split(rng.randint(0, 5000), I2, G)


def _units_and_split(nts, G):
    """Whole-unit waves and the split part's start/length for units with
    nts[u] iterations (units in order)."""
    U = len(nts)
    W = U // G
    D = W * G
    sk0 = sum(nts[:D])
    return W, sk0, sum(nts) - sk0


@pytest.mark.parametrize("seed", range(40))
def test_split_unit_pieces_are_the_ranges_between_its_owners(seed):
    rng = random.Random(1000 + seed)
    G = rng.randint(1, 148)
    nts = [rng.randint(0, 20) for _ in range(rng.randint(1, 3 * G + 5))]
    W, sk0, I2 = _units_and_split(nts, G)
    if I2 == 0:
        return
    U0 = sk0
    covered = []
    for u in range(W * G, len(nts)):
        nt = nts[u]
        if nt == 0:
            continue
        lo, hi = owner(U0, sk0, I2, G), owner(U0 + nt - 1, sk0, I2, G)
        pieces = []
        for c in range(lo, hi + 1):
            a, b = begin(c, sk0, I2, G), begin(c + 1, sk0, I2, G)
            if a < b:   # empty ranges between the owners hold no piece
                s, e = max(a, U0), min(b, U0 + nt)
                assert s < e
                pieces.append((s, e))
        # the pieces tile the unit's iterations in order
        assert pieces[0][0] == U0 and pieces[-1][1] == U0 + nt
        for (a0, a1), (b0, _) in zip(pieces, pieces[1:]):
            assert a1 == b0
        # no CTA outside [lo, hi] touches the unit
        for c in list(range(0, lo)) + list(range(hi + 1, G)):
            a, b = begin(c, sk0, I2, G), begin(c + 1, sk0, I2, G)
            assert b <= U0 or a >= U0 + nt
        covered.extend((s, e, U0, nt) for s, e in pieces)
        U0 += nt
    assert U0 == sk0 + I2
    assert sum(e - s for s, e, _, _ in covered) == I2
    # Partial results: a piece of a unit that other CTAs share goes to one of
    # its CTA's two slots, slot 0 if the unit began at or before the CTA's
    # range (the piece opens the range), else slot 1 (it closes the range).
    # No CTA ever needs the same slot twice.
    for c in range(G):
        a, b = begin(c, sk0, I2, G), begin(c + 1, sk0, I2, G)
        used = []
        for s_, e_, u0, nt in covered:
            if a <= s_ < b and not (s_ == u0 and e_ == u0 + nt):   # a shared unit
                slot = 0 if a >= u0 else 1
                assert (slot == 0 and s_ == a) or (slot == 1 and e_ == b)
                used.append(slot)
        assert len(used) == len(set(used)) <= 2


def test_host_bound_keeps_the_arithmetic_in_32_bits():
    """At the largest call the host lets through (iterations x G just below
    2^31, G = 148), every product the formulas form fits in int32."""
    G = 148
    it_max = (2 ** 31 - 1) // G
    rng = random.Random(7)
    for _ in range(2000):
        I2 = rng.randint(1, it_max)
        sk0 = it_max - I2
        for c in (0, 1, G // 2, G - 1, G):
            begin(c, sk0, I2, G)
        for x in (sk0, sk0 + I2 // 2, sk0 + I2 - 1):
            c = owner(x, sk0, I2, G)
            assert begin(c, sk0, I2, G) <= x < begin(c + 1, sk0, I2, G)


# --------------------------------------------------------------------------
# Multiply-shift division of the query coordinates: q / d computed as
# (q * m) >> 40 with m = ceil(2^40 / d).  Exact whenever q * d < 2^40, the
# bound the entry point enforces before launching the tensor-core kernel
# (F*T x T, T x Tv, Tv x gw).
# --------------------------------------------------------------------------
def _fastdiv(n, d):
    m = ((1 << 40) + d - 1) // d
    return (n * m) >> 40


@pytest.mark.parametrize("d", [1, 2, 3, 7, 52, 80, 1560, 1564, 3520, 14080, 65535, 1 << 20])
def test_fastdiv_exact_below_the_bound(d):
    rng = random.Random(d)
    n_max = ((1 << 40) - 1) // d   # largest n with n * d < 2^40
    ns = [0, 1, d - 1, d, d + 1, n_max, n_max - 1] + [rng.randint(0, n_max) for _ in range(20000)]
    # every multiple of d and its neighbours near the top of the range
    top = n_max // d * d
    ns += [top - 1, top, min(top + 1, n_max)]
    for n in ns:
        assert _fastdiv(n, d) == n // d, (n, d)


def test_fastdiv_fails_above_the_bound():
    """The bound is needed: past it some quotient comes out one too high."""
    d = 1560 * 64 + 1          # a frame of more than 2^16 tokens
    m = ((1 << 40) + d - 1) // d
    e = m * d - (1 << 40)      # rounding excess of m
    assert e > 0
    # the first multiple-minus-one of d whose excess reaches the next integer
    n = d - 1
    while (n * m) >> 40 == n // d:
        n += d
    assert n * d >= 1 << 40 and _fastdiv(n, d) == n // d + 1
