"""The bounded waits every kernel uses give up instead of hanging.

A wait on an mbarrier that nothing arrives on (the state a lost bulk copy
would leave) must return after its budget, and the report must reach the
workspace's error word, where the first error wins.  The helper kernel in
gpu_wait_probe.cu runs the library's own wait and report functions; it is
compiled for sm_100a at test time.
"""
import ctypes
import os
import subprocess

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LQ_DEVERR_TIMEOUT = 2


@pytest.fixture(scope="module")
def probe(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("waitprobe") / "libwaitprobe.so")
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(ROOT, "recurrent_state_quantization_lq_b200", "csrc"),
           os.path.join(HERE, "gpu_wait_probe.cu"), "-o", out]
    subprocess.run(cmd, check=True, capture_output=True, timeout=300)
    lib = ctypes.CDLL(out)
    lib.lq_test_wait_probe.argtypes = [ctypes.c_longlong, ctypes.POINTER(ctypes.c_longlong)]
    lib.lq_test_wait_probe.restype = ctypes.c_int
    return lib


def test_wait_gives_up_after_its_budget_and_reports(probe):
    budget = 2_000_000                        # SM clocks: about a millisecond
    res = (ctypes.c_longlong * 6)()
    assert probe.lq_test_wait_probe(budget, res) == 0
    done, never, waited, code, unit, detail = list(res)
    assert done == 1                          # the completed phase is seen at once
    assert never == 0                         # the empty barrier's wait ran out
    assert budget < waited < 100 * budget     # after the budget, not long after
    assert (code, unit, detail) == (LQ_DEVERR_TIMEOUT, 11, 22)   # first report kept


def test_device_context_usable_after_a_timeout(probe):
    import torch
    res = (ctypes.c_longlong * 6)()
    assert probe.lq_test_wait_probe(1_000_000, res) == 0
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == 1023 * 1024 / 2
