import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an NVIDIA B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")


def build_library():
    """Builds libvlaq.so if stale; build.py is loaded by path so that the
    package (which loads the library on import) is imported only after."""
    import importlib.util
    path = os.path.join(ROOT, "vlaq_quantize_act_b200", "build.py")
    spec = importlib.util.spec_from_file_location("vlaq_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()
