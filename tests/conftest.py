import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU check")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle


@pytest.fixture(scope="session")
def sweep_lib(tmp_path_factory, orc):
    """The exhaustive-sweep helper (tests/native/sweep.c) linked to the oracle."""
    import ctypes
    from oracle import build as ob
    out = tmp_path_factory.mktemp("native") / "libsweep.so"
    src = os.path.join(ROOT, "tests", "native", "sweep.c")
    subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC",
                    src, "-o", str(out), f"-L{ob.OUT_DIR}", "-loracle",
                    f"-Wl,-rpath,{ob.OUT_DIR}", "-lm"], check=True)
    L = ctypes.CDLL(str(out))
    for name in ("sweep_e2m1", "sweep_e4m3"):
        f = getattr(L, name)
        f.restype = ctypes.c_long
        f.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.POINTER(ctypes.c_uint32)]
    return L
