import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large sizes")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def _debug_library_checks(request):
    """With QSA_DEBUG=1 (the debug library, device bounds checks and canary guards), every GPU test
    also ends with no device check fired and every canary guard after a binding-allocated buffer
    intact.  Without it this fixture does nothing."""
    yield
    if os.environ.get("QSA_DEBUG", "0") in ("", "0") or request.node.get_closest_marker("gpu") is None:
        return
    from hybrid_sparse_attention_qsa_b200 import qsa as Q
    Q.qsa_check_canaries()
    status = Q.qsa_get_device_status()
    # tests that plant out-of-range entries read the status themselves; what is left must not be a
    # failed device check
    assert status != Q.QSA_ERR_DEVICE_CHECK, "a device-side bounds check failed"
