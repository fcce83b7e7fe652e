import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


def pytest_sessionstart(session):
    # The shared library is a build artefact (not committed): build it in-tree
    # once per session when it is missing or older than its sources.
    from linear_compressed_attention_b200 import build
    build.build()
