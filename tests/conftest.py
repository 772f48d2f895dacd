import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_sessionfinish(session, exitstatus):
    """Write the parity margins recorded by kda_testlib.assert_close when
    KDA_PARITY_LOG names a file."""
    path = os.environ.get("KDA_PARITY_LOG")
    if not path:
        return
    try:
        import kda_testlib
    except ImportError:
        return
    import json
    with open(path, "w") as f:
        json.dump(kda_testlib.PARITY_LOG, f, indent=1)
