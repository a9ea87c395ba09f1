import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes of CPU oracle time)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    """List both error measures of every parity comparison the session made:
    the normwise max (the asserted one) and the elementwise one."""
    mod = sys.modules.get("gpu_util")
    log = getattr(mod, "ERROR_LOG", None) if mod is not None else None
    if not log:
        return
    per_test = {}
    for test, n, norm, elem in log:
        cnt, tn, mx_norm, mx_elem = per_test.get(test, (0, 0, 0.0, 0.0))
        per_test[test] = (cnt + 1, tn + n, max(mx_norm, norm), max(mx_elem, elem))
    tr = terminalreporter
    tr.section("parity errors (normwise max | elementwise max, per test)")
    for test, (cnt, tn, norm, elem) in sorted(per_test.items()):
        tr.write_line(f"{norm:10.3e} | {elem:10.3e}  {cnt:3d} cmp {tn:12d} el  {test}")
    path = os.environ.get("TTT_ERR_REPORT")
    if path:
        import json
        with open(path, "w") as f:
            json.dump([{"test": t, "comparisons": c, "elements": n, "normwise_max": a, "elementwise_max": b}
                       for t, (c, n, a, b) in sorted(per_test.items())], f, indent=1)
