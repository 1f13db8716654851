"""The split-KV schedule's rules, restated on the host and checked for the properties the kernels rely on.

The attention kernels and the combine each derive the same partition from seq_lens on the device
(tpla_internal.cuh): units (sequence, shard, 64-token page) in b-major order, each weighted by its
sequence's cost (short sequences cost more on the tcgen05 kernels); worker w takes the units whose
weighted start lies in [floor(w V / W), floor((w + 1) V / W)); a segment (one (b, s) run inside a worker)
writes its partial to the pair's own slot W + b g + s when it starts at tile 0, else to the worker's slot.
The combine finds each pair's first and last worker from weighted prefix sums and reads the pair's slot,
then the workers' slots in between.  This restatement checks, over random length mixes and worker
counts, that the rule the combine uses names exactly the segments the attention writes, that no slot is
written twice, and that the weighting evens the cost per worker.  The device code itself is checked on
the GPU (split-schedule invariance and mixed-length parity tests).
"""

import random

import pytest

PAGE = 64


def units_of(lens, gc, max_pages):
    out = []                                   # (b, s, tile, weight) in unit order
    for b, T in enumerate(lens):
        T = max(0, min(T, max_pages * PAGE))
        n = (T + PAGE - 1) // PAGE
        for s in range(gc):
            for t in range(n):
                out.append((b, s, t))
    return out


def weights(lens, w_long, w_short, short_below):
    return [w_short if T < short_below else w_long for T in lens]


def partition(lens, gc, W, wts, max_pages):
    """Attention side: each worker's unit range [lo, hi)."""
    us = units_of(lens, gc, max_pages)
    vpos, v = [], 0
    for (b, s, t) in us:
        vpos.append(v)
        v += wts[b]
    V = v
    ranges = []
    for w in range(W):
        vlo, vhi = w * V // W, (w + 1) * V // W
        lo = next((i for i, x in enumerate(vpos) if x >= vlo), len(us))
        hi = next((i for i, x in enumerate(vpos) if x >= vhi), len(us))
        ranges.append((lo, hi))
    return us, vpos, V, ranges


def writes(us, ranges, gc, W):
    """Slots the attention writes: {slot: (b, s, first unit, last unit)}; empty workers write lse = -inf."""
    slots = {}
    for w, (lo, hi) in enumerate(ranges):
        if lo >= hi:
            assert w not in slots
            slots[w] = None                    # the zero-weight partial
            continue
        i = lo
        while i < hi:
            b, s, t = us[i]
            j = i
            while j + 1 < hi and us[j + 1][:2] == (b, s):
                j += 1
            slot = W + b * gc + s if t == 0 else w
            assert slot not in slots, "slot written twice"
            slots[slot] = (b, s, i, j)
            i = j + 1
    return slots


def combine_reads(lens, gc, W, wts, V, max_pages):
    """Combine side: for each pair, the slots it merges (first: the pair's own slot, then workers)."""
    reads = {}
    vb = 0
    for b, T in enumerate(lens):
        T = max(0, min(T, max_pages * PAGE))
        nt = (T + PAGE - 1) // PAGE
        c = wts[b]
        for s in range(gc):
            if nt:
                v0 = vb + s * nt * c
                worker = lambda v: ((v + 1) * W - 1) // V
                wf, wl = worker(v0), worker(v0 + (nt - 1) * c)
                reads[(b, s)] = [W + b * gc + s] + list(range(wf + 1, wl + 1))
        vb += gc * nt * c
    return reads


CASES = [
    ([32768] * 16, 1, 144),
    ([300, 70, 129, 0, 1], 2, 7),
    ([0, 1, 63, 64, 65, 200, 7, 129], 2, 3),
]


def _random_case(seed):
    rng = random.Random(seed)
    B = rng.randint(1, 40)
    lens = [rng.choice([0, rng.randint(1, 9000), rng.randint(8192, 70000)]) for _ in range(B)]
    return lens, rng.choice([1, 2, 4]), rng.randint(1, 160)


@pytest.mark.parametrize("case", CASES + [_random_case(i) for i in range(40)])
@pytest.mark.parametrize("wts_rule", [(3, 4, 8192), (1, 1, 0)])
def test_combine_reads_exactly_what_the_attention_writes(case, wts_rule):
    lens, gc, W = case
    max_pages = max(1, (max(lens) + PAGE - 1) // PAGE)
    wts = weights(lens, *wts_rule)
    us, vpos, V, ranges = partition(lens, gc, W, wts, max_pages)
    if V == 0:
        return
    # contiguous cover of all units
    assert ranges[0][0] == 0 and ranges[-1][1] == len(us)
    for (lo, hi), (lo2, _) in zip(ranges, ranges[1:]):
        assert hi == lo2 and lo <= hi
    slots = writes(us, ranges, gc, W)
    reads = combine_reads(lens, gc, W, wts, V, max_pages)
    covered = {}
    for (b, s), rs in reads.items():
        first, rest = rs[0], rs[1:]
        assert slots[first] is not None and slots[first][:2] == (b, s)
        got = [slots[first]]
        for k in rest:
            if slots.get(k) is None:           # an empty worker: weight 0
                assert k in slots
                continue
            assert slots[k][:2] == (b, s), "the combine reads another pair's partial"
            got.append(slots[k])
        # the segments read tile the pair's units exactly once, in order
        units = [u for seg in got for u in range(seg[2], seg[3] + 1)]
        assert units == sorted(units) and len(units) == len(set(units))
        assert [us[u][:2] for u in units] == [(b, s)] * len(units)
        assert len(units) == sum(1 for x in us if x[:2] == (b, s))
        covered[(b, s)] = True
    # every written partial is read by its pair
    for slot, seg in slots.items():
        if seg is not None:
            assert (seg[0], seg[1]) in covered


def test_weighting_evens_the_cost_per_worker():
    # 64 sequences of mixed length; tiles of sequences below 8192 tokens cost 4/3 as much
    rng = random.Random(6)
    lens = [rng.randint(1024, 65536) for _ in range(64)]
    gc, W, max_pages = 1, 148, 1024
    cost = lambda b: 4 if lens[b] < 8192 else 3
    for rule in ((1, 1, 0), (3, 4, 8192)):
        wts = weights(lens, *rule)
        us, _, _, ranges = partition(lens, gc, W, wts, max_pages)
        per = [sum(cost(us[i][0]) for i in range(lo, hi)) for lo, hi in ranges]
        spread = max(per) / (sum(per) / W)
        if rule[0] == 1:
            unweighted = spread
        else:
            assert spread <= unweighted and spread < 1.02
