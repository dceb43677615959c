"""The 16-head kernel's work split, replayed on the host with the kernel's
integer rules, on many random batches.

The kernel (decode_attention_qk_b200/csrc/qda_decode_kernel.cu) orders all
pages of the batch sequence by sequence (seg[b] = first page of sequence b),
gives CTA g the pages [g * per_cta, min((g + 1) * per_cta, total)) with
per_cta = ceil(total / grid), and calls the pages of one sequence inside one
CTA a piece. A piece of a sequence split over several CTAs writes its partial
to scratch slot g + b, row ((j * (grid + batch) + slot) * 2 + hb) for kv head
j and query head 2j + hb; the merge of sequence b reads the slots
first + b .. first + b + n - 1, first = seg[b] // per_cta, as one contiguous
block of rows per kv head. What this checks is what those rules promise:
every page is read exactly once, every piece sits in the CTA the merge expects,
slots never collide, the rows of a sequence's pieces are contiguous per kv
head, and every row stays inside the workspace of grid + max_batch slots.
"""
import bisect
import random

PAGE = 16
KV_HEADS = 8
GROUP = 2


def split(lens, grid, stride, max_seq_len=40960):
    """Pages per sequence, the page offsets and per_cta, as the kernel forms them."""
    n = [(L + PAGE - 1) // PAGE if 1 <= L <= max_seq_len and L <= PAGE * stride else 0 for L in lens]
    seg = [0]
    for x in n:
        seg.append(seg[-1] + x)
    total = seg[-1]
    per_cta = (total + grid - 1) // grid if total else 1
    return seg, total, per_cta


def pieces(seg, total, per_cta, grid):
    """(cta, sequence) -> the [first, end) pages of that sequence in that CTA's range."""
    out = {}
    for g in range(grid):
        page, end = g * per_cta, min((g + 1) * per_cta, total)
        while page < end:
            b = bisect.bisect_right(seg, page) - 1   # the sequence holding this page
            stop = min(end, seg[b + 1])
            out[(g, b)] = (page, stop)
            page = stop
    return out


def part_row(j, slot, hb, grid, batch):
    return (j * (grid + batch) + slot) * GROUP + hb


def check(lens, grid, stride, max_batch):
    B = len(lens)
    seg, total, per_cta = split(lens, grid, stride)
    got = pieces(seg, total, per_cta, grid)
    # every page exactly once: the pieces tile [0, total) and each lies inside its sequence
    spans = sorted(got.values())
    if spans:
        assert [a for a, _ in spans] == [0] + [e for _, e in spans[:-1]] and spans[-1][1] == total
    else:
        assert total == 0
    for (g, b), (a, e) in got.items():
        assert seg[b] <= a < e <= seg[b + 1]
    slots = {}
    for b in range(B):
        if seg[b + 1] == seg[b]:
            assert not any(k[1] == b for k in got)
            continue
        first = seg[b] // per_cta
        last = (seg[b + 1] - 1) // per_cta
        holders = sorted(g for (g, bb) in got if bb == b)
        assert holders == list(range(first, last + 1))
        if first == last:
            continue  # whole in one CTA: writes o, no slot
        for g in holders:
            slot = g + b
            assert slot not in slots, (slot, slots.get(slot), (g, b))
            slots[slot] = (g, b)
            assert slot < grid + B <= grid + max_batch
        for j in range(KV_HEADS):
            rows = [part_row(j, first + b + t, hb, grid, B) for t in range(last - first + 1) for hb in range(GROUP)]
            assert rows == list(range(rows[0], rows[0] + len(rows))), "contiguous per kv head"
            assert max(rows) < (grid + max_batch) * KV_HEADS * GROUP, "inside the workspace"


def test_partition_rules_on_random_batches():
    rng = random.Random(20261202)
    for _ in range(3000):
        grid = rng.choice([1, 2, 7, 64, 132, 148, 160])
        max_batch = rng.choice([1, 4, 32, 256])
        B = rng.randint(1, max_batch)
        stride = rng.choice([1, 3, 16, 256, 2560])
        lens = []
        for _ in range(B):
            kind = rng.random()
            if kind < 0.05:
                lens.append(rng.choice([0, -3, PAGE * stride + 1]))  # out of range: no pages
            elif kind < 0.3:
                lens.append(rng.randint(1, 40))
            else:
                lens.append(rng.randint(1, min(40960, PAGE * stride)))
        check(lens, grid, stride, max_batch)


def test_partition_edge_cases():
    check([1], 148, 1, 1)                    # one token
    check([16, 16], 148, 1, 2)               # exactly one page each
    check([40960] * 4, 148, 2560, 4)         # long sequences over many CTAs
    check([17] * 256, 148, 2, 256)           # more sequences than CTAs
    check([40960, 1, 40960], 7, 2560, 3)     # a short sequence between two long ones


# ----------------------------------------------------------------------------
# The chunked prefill's split (decode_attention_qk_b200/csrc/qda_prefill.cu):
# the page-heads of all units (sequence b, kv head j), unit-major, CTA g taking
# [split(g), split(g + 1)), where the running cost (each unit's PIECE_COST
# first, then one per page-head) crosses g * w, w = ceil(W / grid). A piece
# held whole by its CTA writes o; a split unit's pieces write partials to slot
# 2g (the CTA's first piece) or 2g + 1 (its last), and the CTA holding the
# unit's first page records that slot, the one holding its last page its own
# index, for the combine launch, which reads slots first, 2 (g0 + 1), ...,
# 2 gk.

PIECE_COST = 12


def prefill_split(seg, B, grid, g):
    """The kernel's pf_split: the first page-head of CTA g."""
    def cost_before(b):
        return 8 * (seg[b] + PIECE_COST * b)
    W = cost_before(B)
    w = (W + grid - 1) // grid
    t = g * w
    if t >= W:
        return 8 * seg[B]
    lo, hi = 0, B - 1
    while lo < hi:
        mid = (lo + hi + 1) >> 1
        if cost_before(mid) <= t:
            lo = mid
        else:
            hi = mid - 1
    np_ = seg[lo + 1] - seg[lo]
    r = t - cost_before(lo)
    assert r < 8 * (np_ + PIECE_COST)
    j = min(7, r // (np_ + PIECE_COST))
    off = r - j * (np_ + PIECE_COST) - PIECE_COST
    return 8 * seg[lo] + j * np_ + max(0, off)


def prefill_pieces(seg, B, grid):
    """Walk every CTA's range the way the kernel's PieceWalk does; return, per
    unit, the pieces (cta, slot, whole) in order, and what the K producer records."""
    total = 8 * seg[B]
    splits = [prefill_split(seg, B, grid, g) for g in range(grid + 1)]
    units, recorded = {}, {}
    for g in range(grid):
        start, end = splits[g], min(splits[g + 1], total)
        x, k = start, 0
        while x < end:
            b = bisect.bisect_right(seg, x // 8) - 1
            while seg[b + 1] == seg[b]:
                b += 1
            np_ = seg[b + 1] - seg[b]
            r = x - 8 * seg[b]
            j, i0 = r // np_, r % np_
            n = min(np_ - i0, end - x)
            slot = 2 * g + (0 if k == 0 else 1)
            units.setdefault((b, j), []).append((g, slot, i0 == 0 and n == np_, n))
            rec = recorded.setdefault((b, j), [None, None])
            if i0 == 0:
                rec[0] = slot
            if i0 + n == np_:
                rec[1] = g
            x += n
            k += n
    return splits, units, recorded


def test_prefill_split_covers_every_page_head_once_and_the_combine_finds_every_piece():
    rng = random.Random(5)
    for trial in range(2000):
        B = rng.randint(1, 48)
        grid = rng.choice([1, 2, 3, 7, 148, 300])
        pages = [rng.choice([0, 1, 2, 5, 17, 300, 2560]) for _ in range(B)]
        seg = [0]
        for x in pages:
            seg.append(seg[-1] + x)
        total = 8 * seg[B]
        splits, units, recorded = prefill_pieces(seg, B, grid)
        assert splits[0] == 0 and splits[grid] == total
        assert all(splits[i] <= splits[i + 1] for i in range(grid))
        # every page-head in exactly one piece, every unit of a non-empty sequence present
        assert sum(n for lst in units.values() for *_, n in lst) == total
        assert len(units) == 8 * sum(1 for b in range(B) if seg[b + 1] > seg[b])
        for (b, j), lst in units.items():
            assert sum(n for *_, n in lst) == seg[b + 1] - seg[b]
            ctas = [c for c, *_ in lst]
            assert ctas == list(range(ctas[0], ctas[-1] + 1)), "a unit's pieces sit in consecutive CTAs"
            first, last = recorded[(b, j)]
            g0, gk = first >> 1, last
            assert g0 == ctas[0] and gk == ctas[-1]
            if g0 == gk:
                assert len(lst) == 1 and lst[0][2], "a unit in one CTA is written whole"
                continue
            want = [first] + [2 * (g0 + k) for k in range(1, gk - g0 + 1)]
            assert [s for _, s, _, _ in lst] == want, "the combine reads the slots the pieces wrote"
            assert not any(w for _, _, w, _ in lst)
        # slots stay inside the scratch of 2 * grid
        for lst in units.values():
            assert all(0 <= s < 2 * grid for _, s, _, _ in lst)
        # the cost total stays an int32 at the largest batch (256 sequences of 40960 tokens)
        assert 8 * (256 * 2560 + PIECE_COST * 256) < 2 ** 31
