import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built libnvfp4.so")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Report the end-to-end differences of the rotated modes against the oracle."""
    helpers = sys.modules.get("gpu_helpers")
    if helpers is None:
        return
    if helpers.ROTATION_WORST[0]:
        terminalreporter.write_line(
            f"rotated values against the oracle: largest difference {helpers.ROTATION_WORST[0]:.1f} fp32 ulps of "
            f"the group maximum; above the floor, {helpers.ROTATION_WORST[1]:.2e} of the value")
    if not helpers.ROTATED_MISMATCH[1]:
        return
    cb, c, sb, s = helpers.ROTATED_MISMATCH
    terminalreporter.write_line(
        f"rotated modes, end to end against the oracle: {cb} of {c} codes ({cb / c:.2e}) and "
        f"{sb} of {s} scales ({sb / s:.2e}) differ")
