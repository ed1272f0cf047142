"""The GPU parity checks themselves, on the CPU: the near-tie rule must
accept a selection that differs from the oracle's only by blocks whose scores
lie within the 1e-3 band of the threshold, and reject every other kind of
difference (planted here in a fake GPU row)."""
import numpy as np
import pytest

import parity_util as pu

# Earlier blocks 0..7 of a query in block 8, topk = 4 (3 earlier blocks kept).
# Oracle order: 2 (9.0), 5 (5.0), 0 (4.0004) | 6 (4.0), 1 (3.0), ...  -> kept {0, 2, 5}
SCORES = np.array([4.0004, 3.0, 9.0, 1.0, 2.0, 5.0, 4.0, 0.5])
B_OWN, TOPK = 8, 4
REF = [0, 2, 5, 8]


def _check(gpu):
    pu.check_near_tie_row(gpu, REF, SCORES, B_OWN, TOPK, "planted")


def test_accepts_a_swap_inside_the_band():
    _check([2, 5, 6, 8])            # 6 (4.0) for 0 (4.0004): 1e-4 relative


@pytest.mark.parametrize("gpu,why", [
    ([2, 5, 1, 8], "swap outside the band"),           # 1 (3.0) is far below the threshold
    ([0, 2, 8, -1], "a kept block missing"),
    ([0, 2, 5, 7], "own block missing"),
    ([0, 2, 2, 8], "repeated block"),
    ([2, 0, 5, 8], "not ascending"),
    ([0, 2, 5, 9], "block out of range"),
])
def test_rejects_planted_mistakes(gpu, why):
    with pytest.raises(AssertionError):
        _check(gpu)


def test_padding_is_checked():
    scores = np.array([1.0, 2.0])            # b = 2 < topk - 1: all kept, one slot padded
    pu.check_near_tie_row([0, 1, 2, -1], [0, 1, 2, -1], scores, 2, 4)
    with pytest.raises(AssertionError):
        pu.check_near_tie_row([0, 1, 2, 0], [0, 1, 2, -1], scores, 2, 4)


def test_validate_rows_excuses_only_near_ties():
    # One row differs inside the band (gap 1e-4), one outside (gap 0.1).
    q = np.zeros((20, 1, 8))
    q[16, 0] = SCORES                         # token 16, B = 2: block 8, earlier blocks 0..7
    q[17, 0] = SCORES
    # one KV head, 10 blocks; centroid j = e_j, so q . c_j = SCORES[j]
    cents = [np.concatenate([np.eye(8), np.zeros((2, 8))])[None]]
    cu = np.array([0, 20])
    rows = [(16, 0)]
    bad = pu.validate_selection_rows(np.array([[2, 5, 6, 8]]), np.array([REF]), np.array([1e-4]), rows, q, cents, cu,
                                     2, TOPK, "band")
    assert bad == [(16, 0)]
    with pytest.raises(AssertionError):
        pu.validate_selection_rows(np.array([[2, 5, 6, 8]]), np.array([REF]), np.array([0.1]), rows, q, cents, cu,
                                   2, TOPK, "outside")
