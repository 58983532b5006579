"""The wrap-around schedule of the tcgen05 forward (csrc/chunk_tc.cu: sched_shape and the
kernel's piece_at), restated in Python on the host, and the properties the kernel relies on
(no GPU).

With more (batch row, value head) units than SMs, the units' chunks are laid end to end and
cut into runs of L = ceil(units x chunks / SMs) chunk-steps, one per CTA, McNaughton's
wrap-around rule: the unit cut by the end of run i does its first chunks at the start of run
i + 1 and its last chunks at the end of run i, starting from the state the first part leaves.
"""
import pytest


def schedule(units, nc, sms):
    """(L, grid, runs) as the kernel computes them, or None where the kernel keeps one CTA per
    unit. runs[i] lists CTA i's pieces in order: (kind, unit, c0, c1, first step)."""
    if nc == 0 or sms <= 0 or units <= sms:
        return None
    total = units * nc
    L = (total + sms - 1) // sms
    grid = (total + L - 1) // L
    runs = []
    for i in range(grid):
        pos, end, step, pieces = i * L, min((i + 1) * L, total), 0, []
        while pos < end:
            u, cu = pos // nc, pos % nc
            nxt = min(end, (u + 1) * nc)
            ln = nxt - pos
            if cu != 0:
                piece = ("FIRST", u, 0, ln)
            elif ln < nc:
                piece = ("LAST", u, nc - ln, nc)
            else:
                piece = ("WHOLE", u, 0, nc)
            pieces.append(piece + (step,))
            step += ln
            pos = nxt
        runs.append(pieces)
    return L, grid, runs


@pytest.mark.parametrize("units", [149, 160, 192, 200, 320, 1000])
@pytest.mark.parametrize("nc", [1, 2, 3, 7, 32, 64, 256])
def test_schedule_covers_every_chunk_once_and_orders_each_unit(units, nc):
    L, grid, runs = schedule(units, nc, 148)
    assert grid <= 148 and L >= nc   # a unit fits in one run: at most two pieces
    seen = {}
    for i, pieces in enumerate(runs):
        for kind, u, c0, c1, step in pieces:
            for c in range(c0, c1):
                assert (u, c) not in seen
                seen[(u, c)] = (i, step + c - c0)
            if kind == "FIRST":
                # at the start of its run, and its unit's last part ends the previous run
                assert step == 0 and i >= 1
                k, lu, lc0, lc1, lstep = runs[i - 1][-1]
                assert (k, lu, lc0) == ("LAST", u, c1)
                # the first part is done (step c1) before the last part starts (step lstep)
                assert c1 <= lstep
            if kind == "LAST":
                assert runs[i + 1][0][:2] == ("FIRST", u)
    assert len(seen) == units * nc
    for u in range(units):   # within a run, a unit's chunks run on consecutive steps
        for c in range(1, nc):
            (r0, s0), (r1, s1) = seen[(u, c - 1)], seen[(u, c)]
            assert r0 != r1 or s1 == s0 + 1


def test_one_cta_per_unit_without_more_units_than_sms():
    assert schedule(148, 32, 148) is None and schedule(128, 32, 148) is None
    # why: forced on the nanochat shape (128 units of 32 chunks on 148 SMs) a run would be
    # 28 steps, shorter than a unit, which could then span three runs
    total = 128 * 32
    assert (total + 147) // 148 == 28 < 32
