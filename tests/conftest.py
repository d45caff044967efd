import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU work (oracle at full size)")


if os.environ.get("SS_CHECK_ERROR_WORD"):
    import pytest

    @pytest.fixture(autouse=True)
    def _error_word_is_clear(request):
        """Under the checked build: no test may leave the device error word set
        (an out-of-range index, or a bounded wait that gave up), unless it
        provokes that on purpose."""
        yield
        if request.node.get_closest_marker("gpu") is None:
            return
        if "timeout" in request.node.name or "times_out" in request.node.name:
            return
        import selective_state_space_ss_b200 as ss

        assert ss.ss_last_device_error() == ss.SS_OK, "device error word set"
