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


# GPU test files in run order.  Files with parity evidence on a B200 come
# first.  The newer ones follow, from the simplest kernel to the one that chains
# the others.  Under -x a failure in a newer file then never hides the older
# evidence.  A GPU file missing from the list runs after the listed ones but
# before test_zz_no_alloc.py, which stays the very last.
GPU_FILE_ORDER = (
    "test_gpu_edges.py", "test_gpu_fullsize.py", "test_gpu_paged.py", "test_gpu_parity.py",
    "test_gpu_canary.py", "test_gpu_max_batch.py", "test_gpu_share.py",
    "test_gpu_window.py",
    "test_gpu_paged_prefill.py", "test_gpu_policy.py", "test_gpu_backward.py", "test_gpu_index_kl.py",
    "test_gpu_autograd.py", "test_gpu_group_shard.py", "test_gpu_timeout.py", "test_gpu_block_sizes.py",
    "test_gpu_key_split.py", "test_gpu_prefill_fused.py", "test_gpu_short_items.py",
    "test_zz_no_alloc.py",          # the allocation-free entry point: always the last file
)


def pytest_collection_modifyitems(session, config, items):
    rank = {name: i for i, name in enumerate(GPU_FILE_ORDER)}

    def key(item):
        if item.get_closest_marker("gpu") is None:
            return -1                                   # CPU tests keep their place, first
        name = os.path.basename(str(item.fspath))
        if name == GPU_FILE_ORDER[-1]:
            return len(GPU_FILE_ORDER) + 1
        return rank.get(name, len(GPU_FILE_ORDER))
    items.sort(key=key)                                 # stable: order within a file is kept


def max_abs(o, r):
    return float(np.max(np.abs(np.asarray(o, np.float64) - np.asarray(r, np.float64))))


def mean_rel(o, r):
    o = np.asarray(o, np.float64)
    r = np.asarray(r, np.float64)
    return float(np.sum(np.abs(o - r)) / max(np.sum(np.abs(r)), 1e-300))
