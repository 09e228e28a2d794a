"""Pins of the host count of the prefill's conditional-rescale decisions
(oracle/rescale_stats.py) on hand-made scores: with d = 1 and scale = 1 a
row's score is q * k * log2(e), so the block maxima are set by the keys."""
import math

import numpy as np

from oracle.rescale_stats import rescale_counts


def scores_case(c1):
    # 256 rows and keys, q = 1; keys of block 0 are 0, keys of block 1 are c1
    N = 256
    q = np.ones((N, 1), dtype=np.float32)
    k = np.zeros((N, 1), dtype=np.float32)
    k[128:, 0] = c1
    return q, k


def test_tile0_has_no_decisions_tile1_one_per_warp():
    # tile 0 sees block 0 only; tile 1 sees blocks 0 and 1: 4 warps x 1 decision
    dec, grew, resc = rescale_counts(*scores_case(0.0), scale=1.0)
    assert (dec, grew, resc) == (4, 0, 0)


def test_growth_below_threshold_is_not_a_rescale():
    c = 2.0                                   # 2 * log2(e) = 2.9 < 8
    dec, grew, resc = rescale_counts(*scores_case(c), scale=1.0)
    assert (dec, grew, resc) == (4, 4, 0)


def test_growth_past_threshold_rescales():
    c = 10.0                                  # 14.4 > 8
    dec, grew, resc = rescale_counts(*scores_case(c), scale=1.0)
    assert (dec, grew, resc) == (4, 4, 4)


def test_threshold_boundary():
    c = 8.0 / math.log2(math.e)               # exactly 8 in log2 units: not past it
    dec, grew, resc = rescale_counts(*scores_case(c * 0.999), scale=1.0)
    assert resc == 0
    dec, grew, resc = rescale_counts(*scores_case(c * 1.001), scale=1.0)
    assert resc == 4


def test_reference_moves_only_on_a_rescale():
    # three tiles: block 1 raises the max by 9 (rescale), block 2 by 9 more
    # relative to block 1 (another), so tile 2's warps rescale twice
    N = 384
    q = np.ones((N, 1), dtype=np.float32)
    k = np.zeros((N, 1), dtype=np.float32)
    step = 9.0 / math.log2(math.e)
    k[128:256, 0] = step
    k[256:, 0] = 2 * step
    dec, grew, resc = rescale_counts(q, k, scale=1.0)
    # tile 1: 4 decisions (block 1), 4 rescales; tile 2: 8 decisions, 8 rescales
    assert (dec, grew, resc) == (12, 12, 12)
