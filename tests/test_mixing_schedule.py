"""The tensor-core head mixing's copy schedule, checked on the CPU.

Each mixer warp walks its pages' steps in order: 16 unit rows per page, one or two k-steps of 16
sender heads per row (NKT), one 2 KB ring slot per step and kD slots in all; the compute reads step
s from slot s % kD.  Within a page the warp refills the slot it just read with the step kD ahead at
a fixed offset (row + (kt + kD) // NKT, (kt + kD) % NKT); rows from kTail = 16 - ceil(kD / NKT) on
refill through a cursor that resumes at step kTail * NKT + kD of the page and then continues into
the next page's first steps.  This model restates those index formulas (retrieve_tc.cu,
`fetch_static`, `fetch_step`, `sub_step`) and checks that every slot holds the step the compute
reads from it, for every ring depth the shared memory could hold and every mix of page kinds.
"""
from __future__ import annotations

import random

import pytest

ROWS = 16


def simulate(pages, kd):
    """pages: list of NKT values (1 or 2).  Returns the list of (page, row, kt) read at each compute
    step and the slot contents at that moment; raises AssertionError on a mismatch."""
    steps = [(pi, row, kt) for pi, nkt in enumerate(pages) for row in range(ROWS) for kt in range(nkt)]
    slot_of = {}            # slot -> step it holds
    # cursor: (page index, step index within the page); prologue copies the first kd steps
    cur_page, cur_s = 0, 0

    def cursor_next():
        nonlocal cur_page, cur_s
        while cur_page < len(pages) and cur_s == ROWS * pages[cur_page]:
            cur_page, cur_s = cur_page + 1, 0
        if cur_page >= len(pages):
            return None
        nkt = pages[cur_page]
        item = (cur_page, cur_s // nkt, cur_s % nkt)
        cur_s += 1
        return item

    issued = 0
    for u in range(kd):
        slot_of[u] = cursor_next()
        issued += 1
    read = []
    g = 0  # global step index
    for pi, nkt in enumerate(pages):
        k_tail = ROWS - (kd + nkt - 1) // nkt
        assert k_tail * nkt + kd <= ROWS * nkt
        # on entry the cursor has copied this page's first kd steps (or fewer pages remain)
        assert cur_page == pi and cur_s == min(kd, ROWS * nkt) or cur_page > pi
        cur_s = k_tail * nkt + kd  # the in-page steps from kd on are fetched statically
        for row in range(ROWS):
            for kt in range(nkt):
                slot = g % kd
                assert slot_of[slot] == (pi, row, kt), (kd, pages, pi, row, kt, slot_of[slot])
                read.append(slot_of[slot])
                if row < k_tail:
                    ahead = kt + kd
                    slot_of[slot] = (pi, row + ahead // nkt, ahead % nkt)
                else:
                    slot_of[slot] = cursor_next()
                g += 1
    assert read == steps
    return read


@pytest.mark.parametrize("kd", [2, 3, 4, 5, 6, 7, 8])
def test_every_slot_holds_the_step_read_from_it(kd):
    rng = random.Random(1234 + kd)
    for _ in range(200):
        pages = [rng.choice((1, 2)) for _ in range(rng.randint(1, 9))]
        simulate(pages, kd)


def test_static_offsets_stay_inside_the_page():
    # the fixed-offset refill of a non-tail row never leaves its page
    for kd in range(2, 9):
        for nkt in (1, 2):
            k_tail = ROWS - (kd + nkt - 1) // nkt
            for row in range(k_tail):
                for kt in range(nkt):
                    ahead = kt + kd
                    assert row + ahead // nkt < ROWS
