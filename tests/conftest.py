import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


# Config-level parity tests build a full-size step and its oracle once per config and keep only
# the current one; running every test of one config before the next avoids rebuilding them.
CONFIG_ORDER = ["tiny_decode", "llama8b_decode", "mixed_step", "prefix_share_decode",
                "long70b_decode", "long70b_decode_fp8", "mixed_step_fp8"]


def pytest_collection_modifyitems(session, config, items):
    slots = [i for i, it in enumerate(items)
             if it.nodeid.startswith("tests/test_gpu_parity.py")
             and getattr(it, "callspec", None) is not None and "name" in it.callspec.params]
    if not slots:
        return
    group = sorted((items[i] for i in slots),
                   key=lambda it: CONFIG_ORDER.index(it.callspec.params["name"])
                   if it.callspec.params["name"] in CONFIG_ORDER else len(CONFIG_ORDER))
    for i, it in zip(slots, group):
        items[i] = it


def golden_lines(name):
    """Non-comment, non-empty lines of a golden fixture, split on whitespace."""
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle
