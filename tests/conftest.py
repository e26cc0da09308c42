import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# Output tolerance of the main branch against the fp64 oracle: max-abs 2e-2 and
# mean-relative 5e-3, mean-relative being sum|o - r| / sum|r| over all compared
# elements.  Selections (integer block ids) must match exactly.
MAX_ABS_TOL = 2e-2
MEAN_REL_TOL = 5e-3


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def max_abs(o, r):
    return float(np.max(np.abs(np.asarray(o, np.float64) - np.asarray(r, np.float64))))


def mean_rel(o, r):
    o = np.asarray(o, np.float64)
    r = np.asarray(r, np.float64)
    return float(np.sum(np.abs(o - r)) / max(np.sum(np.abs(r)), 1e-300))
