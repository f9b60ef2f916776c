import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


def pytest_sessionstart(session):
    """(Re)build libpaged_attn.so in-tree when it is missing or older than its sources (incremental; the
    binding refuses to import without it)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("_pa_build", os.path.join(ROOT, "paged_kv_cache_330_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
