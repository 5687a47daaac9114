import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200) and the built library")
    config.addinivalue_line("markers", "slow: full-size workloads")


def pytest_sessionstart(session):
    # The library is a build artefact (not committed): compile it if missing or stale.
    from paged_kv_cache_350_b200.build import build
    build()
