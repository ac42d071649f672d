import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.default()


def load_golden(name):
    import json
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def closed_form(expr: str) -> float:
    """Evaluate a closed-form expression from a golden file with math only."""
    import math
    env = {k: getattr(math, k) for k in ("sqrt", "exp", "cos", "sin", "pi", "log")}
    env["float"] = float
    return float(eval(expr, {"__builtins__": {}}, env))
