import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Rows of a whitespace-separated fixture under tests/golden, comments dropped."""
    rows = []
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


def pytest_runtest_teardown(item, nextitem):
    """Under the bounds-checked build (QLORA_B200_BUILD=debug), every GPU test
    must leave no failed index check behind."""
    if os.environ.get("QLORA_B200_BUILD") != "debug" or item.get_closest_marker("gpu") is None:
        return
    import bit_nf4_quantized_16_b200 as q
    line, unit = q.qlora_debug_bounds()
    assert line == 0, f"bounds check failed at {unit}:{line} during {item.nodeid}"
