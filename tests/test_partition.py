"""The decode kernels' length-balanced partition, checked on the host.

The partition is integer arithmetic that every worker derives from the sequence lengths (both
CTAs of a cluster in the tensor-core kernel; each CTA in the small-head kernel).  The sequences'
costs (pages + a fixed boundary cost: 6 pages for the tensor-core kernel, 1 for the small-head
kernel) are concatenated and cut into U = min(W // s_q, T) equal ranges, W = 74 SM pairs or 296
CTAs, and each range is walked by s_q workers, one per query token.  A row whose pages fall in
one range is computed whole.  A row (b, j) cut across ranges a .. c writes, in range R, partial
slot (R + k) * s_q + j, where k counts the sequences before b that are cut.  The combine then
merges slots (a + k) * s_q + j .. (c + k) * s_q + j with stride s_q.  This file restates that
arithmetic in Python and checks the properties the kernels and the combine rely on:
- every page a row attends is attended exactly once;
- every partial slot has one writer and stays below the workspace's 2 W - 2 slots;
- each cut row's slot range holds exactly its segments.
The GPU parity tests check the device code against the oracle.
"""
import numpy as np
import pytest

# (ranges for s_q = 1, boundary cost in pages) of the two kernels that use the partition: the
# tensor-core kernel (one worker per SM pair) and the small-head kernel (two CTAs per SM)
KERNELS = {"tc": (74, 6), "sh": (2 * 148, 1)}


def worker_of(x, T, U):
    return ((x + 1) * U + T - 1) // T - 1


def attended(L, s_q, j, causal):
    return max(0, min(L, L - s_q + j + 1)) if causal else L


def plan(lengths, s_q=1, causal=False, kernel="tc"):
    """Segments (range, row, first page, end page, slot or None) and per-row (c0, c1)."""
    WORKERS, ROW_COST = KERNELS[kernel]
    n_ranges = max(1, WORKERS // s_q)
    rows_pages = [[(attended(int(L), s_q, j, causal) + 63) // 64 for j in range(s_q)] for L in lengths]
    seq_pages = [rp[-1] for rp in rows_pages]
    cost = [p + ROW_COST if p > 0 else 0 for p in seq_pages]
    T = sum(cost)
    U = min(n_ranges, T)
    segs, rowinfo = [], {}
    S, k = 0, 0
    for b, pb in enumerate(seq_pages):
        first = S + ROW_COST
        for j, pr in enumerate(rows_pages[b]):
            r = b * s_q + j
            if pr == 0:
                rowinfo[r] = (-1, -1)
                continue
            a, c = worker_of(first, T, U), worker_of(first + pr - 1, T, U)
            cut = a != c
            rowinfo[r] = ((a + k) * s_q + j, (c + k) * s_q + j) if cut else (a, a)
            for R in range(a, c + 1):
                w0, w1 = R * T // U, (R + 1) * T // U
                g0, g1 = max(w0, first), min(w1, first + pr)
                assert g1 > g0
                segs.append((R, r, g0 - first, g1 - first, (R + k) * s_q + j if cut else None))
        if pb > 0:
            k += worker_of(first, T, U) != worker_of(first + pb - 1, T, U)
        S += cost[b]
    return segs, rowinfo, U


RNG = np.random.default_rng(0)
CASES = [
    ([1], 1, False), ([64], 1, False), ([65] * 3, 1, False), ([0, 0, 5], 1, False),
    ([8192] * 4, 1, False), ([131072] * 4, 1, False), ([4096] * 32, 1, False), ([1] * 300, 1, False),
    (list(RNG.integers(1024, 8193, 64)), 1, False),
    (list(RNG.integers(512, 4097, 128)), 2, True),
    (list(RNG.integers(0, 300, 1000)), 1, False),
    ([1, 70, 640, 129, 2000, 64], 1, False),
    ([1, 2, 65, 129, 130, 4000], 2, True), ([1, 2, 65, 129, 130, 4000], 3, True),
    (list(RNG.integers(1, 3000, 50)), 4, True), (list(RNG.integers(1, 3000, 50)), 2, False),
    ([500] * 10, 80, True),
]


@pytest.mark.parametrize("kernel", sorted(KERNELS))
@pytest.mark.parametrize("lengths,s_q,causal", CASES, ids=lambda x: str(x)[:24])
def test_partition_covers_each_page_once_with_one_writer_per_slot(lengths, s_q, causal, kernel):
    WORKERS = KERNELS[kernel][0]
    SLOTS = 2 * WORKERS - 2
    segs, rowinfo, U = plan(lengths, s_q, causal, kernel)
    assert U * s_q <= max(WORKERS, s_q)
    covered, slots = {}, {}
    for R, r, lo, hi, slot in segs:
        assert 0 <= R < U
        covered.setdefault(r, []).extend(range(lo, hi))
        if slot is not None:
            assert 0 <= slot < SLOTS
            assert slot not in slots, "two writers of one partial slot"
            slots[slot] = r
    for b, L in enumerate(lengths):
        for j in range(s_q):
            r = b * s_q + j
            pr = (attended(int(L), s_q, j, causal) + 63) // 64
            assert sorted(covered.get(r, [])) == list(range(pr)), f"row {r}: pages not attended exactly once"
            c0, c1 = rowinfo[r]
            mine = sorted(s for s, rr in slots.items() if rr == r)
            if pr == 0:
                assert (c0, c1) == (-1, -1)
            elif c0 == c1:
                assert mine == []  # computed whole, written straight to the output
            else:
                assert mine == list(range(c0, c1 + 1, s_q))


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_query_tokens_of_a_sequence_walk_the_same_pages_side_by_side(kernel):
    # s_q = 2 (non-causal): ranges are per sequence, so workers (R, 0) and (R, 1) attend the
    # same pages of the same sequences in the same order
    segs, _, U = plan(list(RNG.integers(512, 4097, 128)), 2, False, kernel)
    by_worker = {}
    for R, r, lo, hi, _ in segs:
        by_worker.setdefault((R, r % 2), []).append((r // 2, lo, hi))
    for R in range(U):
        assert by_worker[(R, 0)] == by_worker[(R, 1)]


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_partition_slot_bound_when_most_range_boundaries_cut_a_row(kernel):
    # long rows against ranges that drift through them: nearly every range boundary falls in
    # some row's pages, the case that uses the most partial slots
    WORKERS = KERNELS[kernel][0]
    SLOTS = 2 * WORKERS - 2
    worst = 0
    rng = np.random.default_rng(3)
    for s_q in (1, 2, 3):
        n = WORKERS
        for lengths in [[64 * 5] + [64 * 13] * (n - 1), [64 * 40] * (n // 2), [64 * 7, 64 * 200, 64 * 3] * (n // 3)] + [
                list(rng.integers(1, 60 * 64, int(rng.integers(2, 3 * n)))) for _ in range(100)]:
            segs, _, U = plan(lengths, s_q, s_q > 1, kernel)
            used = sorted(s for *_, s in segs if s is not None)
            assert len(used) == len(set(used))
            if used:
                assert used[-1] < SLOTS
                worst = max(worst, used[-1] + 1)
    assert worst > 0.6 * SLOTS  # the bound is approached, not just respected
    # one-page rows are never cut (a range boundary cannot fall inside one page)
    segs, _, _ = plan([1] * 8000, kernel=kernel)
    assert all(s is None for *_, s in segs)
