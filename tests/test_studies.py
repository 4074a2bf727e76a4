"""CPU checks of the host-side arithmetic of the measurement studies."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import lookahead_study  # noqa: E402


def test_stale_split_loads_by_hand():
    # fixed [5, 0, 2]; edge 0 (0 -> 1) had kept 30 % at home, edge 1 (2 -> 1) 50 %;
    # the later step's edges carry 10 and 7 tokens: home keeps 3 and 4 (3.5 rounds to even)
    loads = lookahead_study.stale_loads(np.array([5, 0, 2]), np.array([0, 2]), np.array([1, 1]),
                                        np.array([10, 7]), np.array([0.3, 0.5]))
    assert loads.tolist() == [5 + 3, 7 + 3, 2 + 4]
    assert loads.sum() == 5 + 2 + 10 + 7
