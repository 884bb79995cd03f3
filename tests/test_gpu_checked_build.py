"""The bounds-checked build of the library (liblq_checked.so, compiled with
LQ_BOUNDS_CHECK): its kernels test the indices they derive from workspace
contents, skip an access outside its region and record LQ_DEVERR_BOUNDS in
the error word.  Nothing traps.

Two checks: the parity suites for the ragged phases, the tensor-core pass and
the small decode cases pass unchanged against the checked build (no index is
ever reported in correct operation), and a workspace whose per-unit window
count has been corrupted (as a bad checkpoint restore would leave it) is
reported without the access being made.
"""
import os
import subprocess
import sys

import pytest
import torch

from recurrent_state_quantization_lq_b200 import build as lqbuild
from recurrent_state_quantization_lq_b200 import inputs, lq

from harness import to_device

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEV = "cuda"
IN_CHECKED_BUILD = os.path.abspath(lq.LIB_PATH) == os.path.abspath(lqbuild.LIB_CHECKED)


def _pytest_with_checked_build(*args):
    lqbuild.build(bounds_check=True)
    env = dict(os.environ, LQ_LIBRARY=lqbuild.LIB_CHECKED)
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *args],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)


def test_parity_suites_pass_on_the_checked_build():
    r = _pytest_with_checked_build("-m", "gpu", "tests/test_gpu_ragged.py", "tests/test_gpu_tc_path.py",
                                   "tests/test_gpu_parity.py", "-k",
                                   "ragged or tensor_core or window_decode_variants or naive or fp32_state or partial")
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout


def test_checked_build_reports_a_corrupted_window_count():
    r = _pytest_with_checked_build("-m", "gpu",
                                   "tests/test_gpu_checked_build.py::test_corrupted_count_inside_the_checked_build")
    assert r.returncode == 0 and "1 passed" in r.stdout, r.stdout[-4000:] + r.stderr[-2000:]


@pytest.mark.skipif(not IN_CHECKED_BUILD, reason="runs in a process that loads liblq_checked.so (see above)")
def test_corrupted_count_inside_the_checked_build():
    B, H, d, W = 2, 4, 64, 8
    tb = to_device(inputs.tokens(3, 0, 4, B, H, d, d, per_channel_gate=False), DEV)
    st = lq.DecodeState(B, H, d, window=W, ragged=True, device=DEV)
    st.prefill(None)
    for t in range(3):
        st.decode_step(tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t])
    assert st.device_status() == lq.LQ_OK
    victim = 5                                     # sequence 1, head 1
    st.view("fill").view(-1)[victim] = -3          # an inconsistent state, written into the workspace
    before = st.read("buf_delta", check=False).reshape(B * H, W, d)
    st.decode_step(tb.q[3], tb.k[3], tb.v[3], tb.g[3], tb.beta[3])
    assert st.device_status() == lq.LQ_ERR_DEVICE
    assert "index out of range" in lq.last_error()
    err = st.view("err")[:3].cpu()
    assert int(err[0]) == lq.LQ_DEVERR_BOUNDS and int(err[1]) == victim
    after = st.read("buf_delta", check=False).reshape(B * H, W, d)
    # the victim's token was refused: nothing landed in the slots before its own
    # (the previous unit's last slots), and its count is unchanged
    assert torch.equal(after[victim - 1, W - 3:], before[victim - 1, W - 3:])
    fills = st.fills().reshape(-1)
    assert int(fills[victim]) == -3
    others = [u for u in range(B * H) if u != victim]
    assert (fills[others] == 4).all()
