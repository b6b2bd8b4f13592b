import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size workloads)")


def golden_lines(name):
    """Non-comment, non-empty lines of a golden fixture, split on whitespace."""
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                out.append(line.split())
    return out


@pytest.fixture(scope="session")
def golden():
    return golden_lines


@pytest.fixture(scope="session")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_weight_only_router_b200 import build
    build.build()
    torch.cuda.set_device(0)
    return torch.device("cuda:0")


@pytest.fixture(scope="session")
def layer0(dev):
    """The decode/prefill layer: experts seed 0, router seed 1 (host copies and
    device copies)."""
    import moe_inputs as gen
    import nvfp4_weight_only_router_b200 as lib
    ex = gen.make_experts(0)
    rt = gen.make_router(1)
    return {"ex": ex, "rt": rt, "dex": lib.Experts.from_host(ex, dev), "drt": lib.Router.from_host(rt, dev)}
