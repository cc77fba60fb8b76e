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
    config.addinivalue_line("markers", "slow: long-running check at full configuration sizes")


def _ensure_built():
    """Build libplx.so (nvcc cross-compiles without a GPU) if it is missing."""
    import os
    lib = os.path.join(ROOT, "covariance_corrected_softmax_b200", "libplx.so")
    if not os.path.exists(lib):
        from covariance_corrected_softmax_b200 import build
        build.build()


_ensure_built()
