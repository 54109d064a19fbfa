import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    # a fresh checkout has no built library (it is not versioned): build it once, by
    # the build script's path, before any test module imports the package
    if not os.path.exists(os.path.join(ROOT, "vision_selective_state_b200", "libvscan.so")):
        import __graft_entry__

        __graft_entry__._load_build_script(os.path.join("vision_selective_state_b200", "build.py"),
                                           "_vscan_build").build()


def read_golden(name):
    """Non-comment, non-empty lines of a golden fixture."""
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]


def read_route_fixture(name):
    """{(H, W): {k: [indices]}} from a route fixture."""
    out, cur = {}, None
    for ln in read_golden(name):
        if ln.startswith("grid"):
            h, w = ln.split()[1].split("x")
            cur = (int(h), int(w))
            out[cur] = {}
        else:
            k, rest = ln.split(":")
            out[cur][int(k)] = [int(v) for v in rest.split()]
    return out


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    return oracle
