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
