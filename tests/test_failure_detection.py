"""Failure detection without a GPU fault: every pipeline wait in libgqa is bounded.

A test-only kernel waits, with the library's own bounded wait, on an mbarrier that nothing ever
completes.  The wait must give up after its limit (1 s), set the timeout bit of the error word,
raise the CTA-wide abort flag that the kernel's other roles poll, and return: the kernel ends
normally and the CUDA context stays usable.  The contrasting case completes immediately.
"""
import ctypes
import os
import shutil
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
TIMEOUT_BIT = 2   # GQA_DEVERR_TIMEOUT in include/gqa.h


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    out = str(tmp_path_factory.mktemp("bw") / "libbounded_wait.so")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17", "-shared",
                    "-Xcompiler", "-fPIC", "-o", out, os.path.join(HERE, "cuda", "bounded_wait.cu")],
                   check=True, capture_output=True)
    lib = ctypes.CDLL(out)
    lib.run_wait.argtypes = [ctypes.c_int] + [ctypes.POINTER(ctypes.c_int)] * 3 + [ctypes.POINTER(ctypes.c_float)]
    lib.run_wait.restype = ctypes.c_int
    return lib


def _run(lib, arrive_first):
    ok, ab, err, ms = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_float()
    rc = lib.run_wait(arrive_first, ctypes.byref(ok), ctypes.byref(ab), ctypes.byref(err), ctypes.byref(ms))
    assert rc == 0
    return ok.value, ab.value, err.value, ms.value


def test_wait_that_never_completes_gives_up_and_reports(probe):
    ok, ab, err, ms = _run(probe, 0)
    assert ok == 0
    assert ab == 1
    assert err & TIMEOUT_BIT
    assert 900.0 <= ms <= 10_000.0
    # The context is still usable afterwards.
    x = torch.ones(1024, device="cuda")
    assert float(x.sum().item()) == 1024.0


def test_wait_that_completes_returns_at_once(probe):
    ok, ab, err, ms = _run(probe, 1)
    assert (ok, ab, err) == (1, 0, 0)
    assert ms < 100.0
