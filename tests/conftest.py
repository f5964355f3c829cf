import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an sm_100 (B200) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def _have_sm100():
    try:
        import torch
        if not torch.cuda.is_available():
            return False
        major, _ = torch.cuda.get_device_capability(0)
        return major == 10
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if _have_sm100():
        return
    skip = pytest.mark.skip(reason="no sm_100 GPU in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The raw max-abs error of every output every parity test compared with
    the oracle (bar: 1e-2 on O/dQ/dK/dV, 1e-3 on LSE), the elements excused as
    bf16 output rounding of values >= 4 in magnitude, and the worst raw error
    per output kind over the whole run."""
    gc = sys.modules.get("tests.gpu_common")
    report = getattr(gc, "REPORT", None) if gc is not None else None
    if not report:
        return
    tr = terminalreporter
    tr.section("parity: raw max-abs vs the fp64 oracle")
    worst = {}
    n_exc = 0
    for test, outs in report.items():
        cells = []
        for name, d in outs.items():
            cells.append(f"{name} {d['raw']:.5f}" + (f" ({len(d['excused'])} excused)" if d["excused"] else ""))
            kind = name.split("#")[0].split("[")[0]
            if d["raw"] > worst.get(kind, (-1.0, ""))[0]:
                worst[kind] = (d["raw"], test)
            n_exc += len(d["excused"])
            for ix, ref, err in d["excused"]:
                tr.write_line(f"  excused {test} {name}{list(ix)}: oracle {ref:.5f} error {err:.5f}")
        tr.write_line(f"{test.split('::', 1)[-1]}: " + ", ".join(cells))
    path = os.environ.get("BSA_PARITY_LOG")
    if path:
        try:
            with open(path, "w") as f:
                json.dump(report, f, indent=1)
        except OSError:
            pass
    tr.write_line("worst raw max-abs per output: " + ", ".join(
        f"{k} {v[0]:.5f}" for k, v in sorted(worst.items())) + f"; excused elements {n_exc}")
