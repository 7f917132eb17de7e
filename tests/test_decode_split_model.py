"""Host model of the decode kernel's work split, swept over many shapes.

The kernel flattens (unit, 32-slot chunk) pairs, where a unit is (batch row, kv
head, head chunk), and gives CTA c the contiguous chunks [c W / C, (c + 1) W / C).
Two chunk layouts exist:
  - uniform: every unit has ceil(max kv_len / 32) chunks;
  - per-row: a unit has ceil(kv_len[b] / 32) chunks, placed through a prefix over
    the rows.
A split unit is merged in the kernel from one partial record per owner CTA:
record 2 c for c's first unit and 2 c + 1 for its last.  This model restates the
kernel's integer rules and checks the invariants the merge relies on:
  - every chunk has exactly one owner;
  - the owner count the kernel computes equals the number of CTAs whose range
    meets the unit;
  - a CTA shares at most its first and its last unit;
  - record slots are unique per (CTA, slot);
  - no two split units have the same first owner CTA (the merge counter of a
    split unit is the one of its first owner, at a shape-independent offset).
With one kv_len for every row the kernel may stream with U k of its CT0 CTAs
(k = floor(CT0 / U)) instead of all of them, when that costs a warp no more
rounds of chunks; each CTA's range then lies inside one unit.
"""
import random


def range_start(c, W, C):
    return c * W // C


def cta_of(idx, W, C):
    return ((idx + 1) * C - 1) // W


def active_ctas(U, nch, CT0, NW):
    k = CT0 // U
    if k < 1:
        return CT0
    rounds_all = (-(-U * nch // CT0) + NW - 1) // NW
    rounds_units = (-(-nch // k) + NW - 1) // NW
    return U * k if rounds_units <= rounds_all else CT0


def check_split(lens_per_unit, C):
    starts, W = [], 0
    for n in lens_per_unit:
        starts.append(W)
        W += n
    if W == 0:
        return

    def unit_of(idx):  # the unit whose chunk range holds idx (units with no chunks are skipped)
        lo, hi = 0, len(starts) - 1
        while lo < hi:
            mid = (lo + hi + 1) // 2
            if starts[mid] <= idx:
                lo = mid
            else:
                hi = mid - 1
        while lens_per_unit[lo] == 0:  # several units may share a start; the one with chunks comes last
            lo += 1
        return lo

    # every chunk is owned by the CTA whose range holds it
    for idx in range(W):
        c = cta_of(idx, W, C)
        assert range_start(c, W, C) <= idx < range_start(c + 1, W, C)
    used = set()
    counters = set()
    for u, n in enumerate(lens_per_unit):
        if n == 0:
            continue
        s, e = starts[u], starts[u] + n - 1
        cf, cl = cta_of(s, W, C), cta_of(e, W, C)
        true_owners = sorted({cta_of(i, W, C) for i in range(s, e + 1)})
        if cf == cl:
            assert true_owners == [cf]
            continue
        owners = cl - cf + 1 if W >= C else n  # the kernel's count
        assert owners == len(true_owners), (lens_per_unit, C, u)
        assert cf not in counters, "two split units would share a merge counter"
        assert 0 <= cf < C
        counters.add(cf)
        listed = [cf + o if W >= C else cta_of(s + o, W, C) for o in range(owners)]
        assert listed == true_owners
        for c in listed:
            first = unit_of(range_start(c, W, C))
            last = unit_of(range_start(c + 1, W, C) - 1)
            slot = 0 if u == first else 1
            assert u in (first, last), "a CTA shares only its first and last unit"
            assert (c, slot) not in used
            used.add((c, slot))


def test_uniform_split_invariants():
    rng = random.Random(1)
    for _ in range(400):
        U = rng.randint(1, 80)
        nch = rng.randint(1, 300)
        C = rng.choice([1, 2, 7, 148, 256])
        check_split([nch] * U, C)


def test_per_row_split_invariants():
    rng = random.Random(2)
    for _ in range(400):
        B = rng.randint(1, 40)
        UH = rng.choice([1, 2, 8, 16])  # units per row (kv heads x head chunks)
        rows = [0 if rng.random() < 0.2 else rng.randint(1, 300) for _ in range(B)]
        C = rng.choice([1, 3, 148, 256])
        check_split([n for n in rows for _ in range(UH)], C)


def test_fewer_chunks_than_ctas():
    # one chunk per CTA at most: every split unit has one owner per chunk
    check_split([3, 1, 0, 2], 148)
    check_split([1] * 100, 148)


def test_unit_aligned_grid():
    rng = random.Random(3)
    for _ in range(600):
        U = rng.randint(1, 160)
        nch = rng.randint(1, 400)
        CT0 = rng.choice([132, 148, 256])
        NW = rng.choice([4, 6, 8])
        C = active_ctas(U, nch, CT0, NW)
        assert 1 <= C <= CT0
        check_split([nch] * U, C)
        if C != CT0:
            k = C // U
            assert C == U * k and k == CT0 // U
            W = U * nch
            for c in range(C):  # every CTA's range lies inside unit c // k
                b, e = range_start(c, W, C), range_start(c + 1, W, C)
                if b < e:
                    assert (c // k) * nch <= b and e <= (c // k + 1) * nch
    # the CTAs that stream are spread over the grid: CTA b takes place floor(b CT / CT0)
    # when the next CTA's is larger, and the places are 0 .. CT - 1, once each
    for CT0 in (132, 148):
        for CT in range(1, CT0 + 1):
            places = [b * CT // CT0 for b in range(CT0) if (b + 1) * CT // CT0 > b * CT // CT0]
            assert places == list(range(CT))
    # the decode workload (8 x 8 units, 64 chunks of 64 slots, 8 warps): two CTAs a unit
    assert active_ctas(64, 64, 148, 8) == 128
    # a long single-row decode keeps the flattened split (fewer rounds per warp)
    assert active_ctas(16, 4096, 148, 6) == 148


def row_aligned_split(row_chunks, UH, CT0, NW):
    """The kernel's split for rows of different lengths (at most 32 rows): k_b CTAs a
    unit for row b, one each, then one more at a time to the row with the most chunks
    a CTA (ties: the lower row) while UH * sum(k_b) stays within the grid; used when no
    warp then takes more rounds than with the flattened cut.  Returns the CTAs' chunk
    ranges, or None when the flattened cut is kept."""
    B = len(row_chunks)
    if B > 32 or B * UH > CT0:
        return None
    k = [1 if n > 0 else 0 for n in row_chunks]
    rem = CT0 // UH - sum(k)
    while rem > 0:
        best, who = max(((-(-n // kk) if kk else 0), -b) for b, (n, kk) in enumerate(zip(row_chunks, k)))
        if best <= 1:
            break
        k[-who] += 1
        rem -= 1
    W = UH * sum(row_chunks)
    rounds_all = (-(-W // CT0) + NW - 1) // NW
    mx = max(((-(-n // kk) if kk else 0) + NW - 1) // NW for n, kk in zip(row_chunks, k))
    if mx > rounds_all:
        return None
    ranges, start = [], 0
    for n, kk in zip(row_chunks, k):
        for uu in range(UH):
            us = start + uu * n
            for j in range(kk):
                ranges.append((us + j * n // kk, us + (j + 1) * n // kk))
        start += UH * n
    return ranges


def test_row_aligned_split():
    rng = random.Random(4)
    for _ in range(500):
        B = rng.randint(1, 32)
        UH = rng.choice([1, 2, 4, 8])
        rows = [0 if rng.random() < 0.15 else rng.randint(1, 300) for _ in range(B)]
        NW = rng.choice([6, 8])
        r = row_aligned_split(rows, UH, 148, NW)
        if r is None:
            continue
        assert len(r) <= 148
        covered = sorted(i for b, e in r for i in range(b, e))
        assert covered == list(range(UH * sum(rows)))  # every chunk once
        starts = [0]
        for n in rows:
            for _ in range(UH):
                starts.append(starts[-1] + n)
        for b, e in r:  # a CTA's range lies inside one unit
            if b < e:
                u = max(i for i, s0 in enumerate(starts[:-1]) if s0 <= b and starts[i + 1] > b)
                assert e <= starts[u + 1]
    # the ragged bench batch (8 rows of 512..8192 slots, 64-slot chunks, 8 kv heads)
    r = row_aligned_split([8, 16, 32, 48, 64, 80, 96, 128], 8, 148, 8)
    assert r is not None and len(r) == 144 and max(e - b for b, e in r) == 32
