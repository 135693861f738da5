import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: large CPU oracle work")


def pytest_sessionstart(session):
    # Build the CUDA library (nvcc cross-compiles without a GPU) and the
    # oracle once per session, so that a fresh checkout tests what it builds.
    from quantized_gemm_token_b200 import build as libdq_build
    from oracle import build as oracle_build
    libdq_build.build()
    oracle_build.build()
