"""Host-side checks of the persistent GEMM's tile schedule (no GPU needed).

Every tile must run on exactly one CTA pair, and for the backward launch (a few
long dX tiles with K = V next to many short dW tiles) the k-steps per pair must
be balanced to within one long tile's share of the ideal.
"""
import pytest

import rl_post_policy_b200 as pl


def loads(t0, t1, c0, c1, pairs):
    rc, owner = pl.pl_debug_pair_tiles(t0, t1, c0, c1, pairs)
    assert rc == 0
    per = [0] * pairs
    for t, q in enumerate(owner):
        per[q] += c0 if t < t0 else c1
    return per


@pytest.mark.parametrize("t0,t1,c0,c1,pairs", [
    (64, 8016, 2004, 16, 74),   # batch-1 backward: 64 dX tiles (K=128256), 8016 dW tiles (K=1024)
    (64, 9504, 2376, 16, 74),   # V=152064, H=4000
    (64, 8016, 2004, 16, 70),   # fewer resident pairs than SM pairs
    (4, 9504, 2376, 4, 74),     # 256-row chunk
    (1, 4, 16, 2, 5),
    (3, 5, 40, 1, 4),
    (10, 10, 1, 1, 3),          # equal costs: round-robin
    (0, 7, 1, 1, 3),
])
def test_every_tile_runs_once(t0, t1, c0, c1, pairs):
    per = loads(t0, t1, c0, c1, pairs)
    assert sum(per) == t0 * c0 + t1 * c1


def test_backward_schedule_is_balanced():
    t0, t1, c0, c1, pairs = 64, 8016, 2004, 16, 74
    per = loads(t0, t1, c0, c1, pairs)
    ideal = (t0 * c0 + t1 * c1) / pairs
    assert max(per) <= ideal + c1        # within one short tile of the ideal
    # plain round-robin would leave the dX pairs ~8% over the ideal
    rr = [0] * pairs
    for t in range(t0 + t1):
        rr[t % pairs] += c0 if t < t0 else c1
    assert max(per) < max(rr)
