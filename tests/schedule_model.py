"""A host restatement of the scheduler's documented rules, for checking the tile ledger the
device reports (``pa_schedule_stats``) and for the CPU tests of the grouping rule.

Rules (from the scheduler's description in ``include/packattn.h``, ``pa_set_short_packing``):
  * a segment of at most 128 tokens is short; with short-segment packing on, runs of
    consecutive short segments are cut greedily, in packing order, into tiles of at most
    128 tokens holding whole segments; a run is also cut where a segment starts in a later
    1024-token block of the stream than the segment before it;
  * two neighbouring tiles of a run form one unit (a group), one work item per head; a unit
    that would hold a single segment leaves that segment alone;
  * every other non-empty segment is a unit of its own with heads * ceil(L / 256) items;
  * score tiles computed: ceil(L/128)^2 per head for a segment alone, one per tile of a group.
Test infrastructure only; it shares no code with the CUDA path.
"""
import math

TILE = 128
BLOCK_LOG2 = 10


def units(lengths, short_packing=True):
    """Units of a pack: ("alone", seg, L) or ("group", first_seg, n0, len, segs)."""
    lengths = [int(n) for n in lengths]
    B = len(lengths)
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + n)
    out = []
    if not short_packing:
        return [("alone", i, n) for i, n in enumerate(lengths) if n > 0]

    def short(i):
        return lengths[i] <= TILE

    def new_block(i):
        return (cu[i - 1] >> BLOCK_LOG2) != (cu[i] >> BLOCK_LOG2)

    def continues(j):  # segment j joins the run of segment j - 1
        return j < B and short(j) and not new_block(j)

    def tile_end(i):
        j = i + 1
        while continues(j) and cu[j + 1] - cu[i] <= TILE:
            j += 1
        return j

    for i in range(B):
        if not short(i):
            out.append(("alone", i, lengths[i]))
            continue
        if i > 0 and short(i - 1) and not new_block(i):
            continue  # inside the run of an earlier segment
        s = i
        while True:
            e1 = tile_end(s)
            e2 = tile_end(e1) if continues(e1) else e1
            n0, ln = cu[e1] - cu[s], cu[e2] - cu[s]
            if ln > 0 and e2 == s + 1:
                out.append(("alone", s, lengths[s]))  # a group of one segment: the segment alone
            elif ln > 0:
                out.append(("group", s, n0, ln, list(range(s, e2))))
            if not continues(e2):
                break
            s = e2
    return out


def ledger(lengths, heads, short_packing=True):
    """(items, units, score_tiles, useful_pairs, groups, grouped_segments) of a forward call."""
    us = units(lengths, short_packing)
    items = tiles = groups = 0
    for u in us:
        if u[0] == "alone":
            items += heads * math.ceil(u[2] / 256)
            tiles += heads * math.ceil(u[2] / TILE) ** 2
        else:
            items += heads
            tiles += heads * (2 if u[3] > u[2] else 1)
            groups += 1
    grouped = sum(1 for u in us if u[0] == "group" for i in u[4] if lengths[i] > 0)
    pairs = heads * sum(int(n) * int(n) for n in lengths)
    return dict(items=items, units=len(us), score_tiles=tiles, useful_pairs=pairs, groups=groups,
                grouped_segments=grouped)
