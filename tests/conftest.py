import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built libsqa")
    # The package refuses to import without its library: build it first (a no-op
    # when it is current). build.py is loaded by path so the package is not imported.
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_sqa_build", os.path.join(ROOT, "reduced_query_head_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    mod.build(debug=True)
