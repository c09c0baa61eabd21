import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running check")


def pytest_collection_modifyitems(config, items):
    # GPU tests need a device; without one they are skipped, never silently
    # routed elsewhere.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


# full-size workloads whose measured errors are printed at the end of a run
_REPORTED = ("test_decode_workloads_full_parity", "test_short_query_workload_full_parity",
             "test_continuous_batching_one_graph_many_steps", "test_prefill_workload_sampled",
             "test_paged_ragged_workload_sampled", "test_noalloc")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Measured parity errors against the oracle (max-abs out, max per-row
    relative out error, max-abs lse) for the full-size workloads."""
    try:
        import gpu_helpers
    except Exception:
        return
    rows = [(k, v) for k, v in sorted(gpu_helpers.ERRORS.items()) if any(r in k for r in _REPORTED)]
    if not rows:
        return
    tr = terminalreporter
    tr.write_line("parity errors vs the fp64 oracle (rows checked, max|out err|, max row rel err, max|lse err|):")
    for k, (n, eo, ro, el) in rows:
        name = k.split("::")[-1]
        tr.write_line(f"  {name}: {n} rows, {eo:.3g}, {ro:.3g}, {el:.3g}")
