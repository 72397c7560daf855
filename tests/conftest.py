import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    # The built library is not committed, and one carried over from another
    # checkout may predate its sources: rebuild whenever any source is newer
    # than liblcsa.so (loaded by path, since importing the package needs the
    # library).
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "lcsa_build", os.path.join(ROOT, "block_sparse_causal_lcsa_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
