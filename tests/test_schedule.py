"""Host-side checks of the persistent GEMM's tile schedule (no GPU needed).

Every tile must run on exactly one CTA pair, and for the backward launch (a few
long dX tiles with K = V next to many short dW tiles) the load per pair -- each
tile's k-steps plus the fixed hand-off cost of 8 k-steps the schedule counts --
must be balanced to within one short tile of the ideal.  The backward launch's
K split of its dX problem runs only when asked for.
"""
import pytest

import rl_post_policy_b200 as pl

HANDOFF = 8  # k-steps the schedule adds per tile


def loads(t0, t1, c0, c1, pairs, handoff=HANDOFF):
    rc, owner = pl.pl_debug_pair_tiles(t0, t1, c0, c1, pairs)
    assert rc == 0
    per = [0] * pairs
    for t, q in enumerate(owner):
        per[q] += (c0 if t < t0 else c1) + handoff
    return per


@pytest.mark.parametrize("t0,t1,c0,c1,pairs", [
    (64, 8016, 2004, 16, 74),   # batch-1 backward: 64 dX tiles (K=128256), 8016 dW tiles (K=1024)
    (32, 4008, 4008, 32, 74),   # the same at 512-wide tiles (k-steps counted per N=256 MMA group)
    (32, 4752, 4752, 32, 74),   # V=152064, H=4000 at 512 wide
    (64, 9504, 2376, 16, 74),   # V=152064, H=4000
    (64, 8016, 2004, 16, 70),   # fewer resident pairs than SM pairs
    (4, 9504, 2376, 4, 74),     # 256-row chunk
    (1, 4, 16, 2, 5),
    (3, 5, 40, 1, 4),
    (10, 10, 1, 1, 3),          # equal costs: round-robin
    (0, 7, 1, 1, 3),
])
def test_every_tile_runs_once(t0, t1, c0, c1, pairs):
    per = loads(t0, t1, c0, c1, pairs, handoff=0)
    assert sum(per) == t0 * c0 + t1 * c1


@pytest.mark.parametrize("t0,t1,c0,c1", [
    (64, 8016, 2004, 16),    # 256-wide backward of a 1024-row chunk
    (64, 4008, 2004, 32),    # 512-wide, dX split in two K halves (k-steps per N=256 MMA group)
    (64, 4752, 2376, 32),    # the same at V=152064, H=4000
])
def test_backward_schedule_is_balanced(t0, t1, c0, c1):
    pairs = 74
    per = loads(t0, t1, c0, c1, pairs)
    ideal = (t0 * (c0 + HANDOFF) + t1 * (c1 + HANDOFF)) / pairs
    assert max(per) <= ideal + c1 + HANDOFF        # within one short tile of the ideal
    # plain round-robin would leave the dX pairs over the ideal
    rr = [0] * pairs
    for t in range(t0 + t1):
        rr[t % pairs] += (c0 if t < t0 else c1) + HANDOFF
    assert max(per) < max(rr)


@pytest.mark.parametrize("name,problems,want", [
    ("forward, 1024 rows", [(1024, 128256, 4096)] * 2, 2),
    ("backward, 1024-row chunk", [(1024, 4096, 128256), (128256, 4096, 1024)], 2),
    ("backward, whole 8192-row batch", [(8192, 4096, 128256), (128256, 4096, 8192)], 2),
    ("backward, 1024-row chunk, V=152064, H=4000", [(1024, 4000, 152064), (152064, 4000, 1024)], 2),
    ("backward, 256-row chunk: 8 wide dX tiles would hold up the launch", [(256, 4096, 128256), (128256, 4096, 256)], 1),
    ("dX alone: 32 wide tiles on 74 pairs", [(1024, 4096, 128256)], 1),
    ("problem narrower than 512", [(1024, 256, 4096)], 1),
    ("one of two problems narrower than 512", [(1024, 4096, 64), (4096, 448, 1024)], 1),
])
def test_tile_width_choice(name, problems, want):
    assert pl.pl_debug_pick_tile(problems, 74) == want, name


def test_pick_tile_rejects_bad_input():
    assert pl.pl_debug_pick_tile([], 74) == -1
    assert pl.pl_debug_pick_tile([(1, 1, 1)] * 3, 74) == -1
    assert pl.pl_debug_pick_tile([(0, 512, 64)], 74) == -1
    assert pl.pl_debug_pick_tile([(256, 512, 64)], 0) == -1


def test_wide_backward_schedule_is_within_one_short_tile_of_its_longest_tile():
    # without the K split, a 512-wide dX tile (4008 units) exceeds the fair share (about
    # 3900 with the hand-off cost): the makespan cannot go below one dX tile, and the
    # schedule stays within one dW tile of it
    t0, t1, c0, c1, pairs = 32, 4008, 4008, 32, 74
    per = loads(t0, t1, c0, c1, pairs)
    assert max(per) <= c0 + c1 + 2 * HANDOFF
    rest = per[t0:]
    assert max(rest) - min(rest) <= c1 + HANDOFF


@pytest.mark.parametrize("name,problems,want_nh", [
    ("1024-row chunk", [(1024, 4096, 128256), (128256, 4096, 1024)], 2),
    ("1024-row chunk, V=152064, H=4000", [(1024, 4000, 152064), (152064, 4000, 1024)], 2),
    ("whole 8192-row batch", [(8192, 4096, 128256), (128256, 4096, 8192)], 2),
    ("square", [(4096, 4096, 4096), (4096, 4096, 4096)], 2),
    ("K of one step", [(1024, 1024, 64), (64, 1024, 1024)], 1),
])
def test_backward_k_split_is_off_unless_asked(name, problems, want_nh):
    # measured no faster on the fused backward launch, the split runs only on request
    assert pl.pl_debug_pick_split(problems, 74) == (1, want_nh), name


def test_k_split_knob_forces_either_choice():
    problems = [(1024, 4096, 128256), (128256, 4096, 1024)]
    try:
        assert pl.pl_debug_set_gemm_split(2) == 0
        assert pl.pl_debug_pick_split(problems, 74) == (2, 2)
        assert pl.pl_debug_pick_split([(4096, 4096, 4096), (4096, 4096, 4096)], 74)[0] == 2
        # a single k-step has no halves
        assert pl.pl_debug_pick_split([(1024, 1024, 64), (64, 1024, 1024)], 74)[0] == 1
        assert pl.pl_debug_set_gemm_split(1) == 0
        assert pl.pl_debug_pick_split(problems, 74)[0] == 1
        assert pl.pl_debug_set_gemm_split(3) != 0
    finally:
        pl.pl_debug_set_gemm_split(0)
    assert pl.pl_debug_pick_split([(1, 1, 1)], 74)[0] == -1


@pytest.mark.parametrize("tiles,q_f0,q_w", [
    ([32, 1004, 1004, 4008], 1, 3),   # merged launch: dX, reference and policy forward, dW
    ([64, 1004, 4008], 1, 2),         # the same at beta = 0 (no reference forward)
    ([1004, 1004, 4008], 0, 2),       # no dX
    ([32, 1004, 1004], 1, -1),        # no dW: job order
    ([3, 0, 5, 9], 1, 3),
])
def test_dynamic_queue_order(tiles, q_f0, q_w):
    rc, order = pl.pl_debug_queue_tiles(tiles, q_f0, q_w)
    assert rc == 0
    total = sum(tiles)
    assert sorted(order) == list(range(total))           # every tile exactly once
    lead = sum(tiles[:q_f0])
    assert order[:lead] == list(range(lead))              # the long tiles first, in order
    if q_w < 0:
        assert order == list(range(total))
        return
    f_begin, w_begin = lead, sum(tiles[:q_w])
    rest = order[lead:]
    fw = [t for t in rest if t < w_begin]
    dw = [t for t in rest if t >= w_begin]
    assert fw == sorted(fw) and dw == sorted(dw)          # each kind in its own order
    # spread evenly: every prefix of the rest holds the forward tiles in proportion
    nf, n = len(fw), len(rest)
    seen = 0
    for i, t in enumerate(rest):
        seen += t < w_begin
        assert abs(seen - (i + 1) * nf / n) <= 1.0


def test_dynamic_queue_rejects_bad_input():
    assert pl.pl_debug_queue_tiles([], 0, -1)[0] == -1
    assert pl.pl_debug_queue_tiles([1, 2, 3, 4, 5], 0, -1)[0] == -1
    assert pl.pl_debug_queue_tiles([1, 2], 2, 1)[0] == -1


@pytest.mark.parametrize("tiles,pairs,want", [
    (2008, 74, 10),    # the batch-1 forward at 512 wide: 27 waves and 10 tiles
    (16064, 74, 6),    # a whole 8192-row batch
    (2018, 74, 20),
    (2049, 74, 0),     # 51 tiles in the last wave: halves would not end it sooner
    (148, 74, 0),      # whole waves
    (50, 74, 0),       # a single partial wave
    (10, 1, 0),
])
def test_tail_halves(tiles, pairs, want):
    r = pl.pl_debug_tail_halves(tiles, pairs)
    assert r == want
    if r:
        # full waves, then 2r halves on 2r pairs: the launch ends half a tile after the full waves
        full = tiles - r
        assert full % pairs == 0 and 2 * r <= pairs
