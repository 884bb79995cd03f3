"""Output quality of the INT8 states against the FP32 state on the GPU.

LeapQuant ("LeapQuant: Efficient Linear Attention with Accurate Recurrent
State Quantization", section "Abstract (arXiv)") reports that quantizing the
state per token collapses quality while the windowed scheme with Compensator
Tokens keeps it.  On a planted-outlier state (2 rows and 2 columns x 50) the
windowed decode must stay close to the FP32-state decode and well below the
naive per-token INT8 decode, window by window.
"""
import pytest
import torch

import bench
from recurrent_state_quantization_lq_b200 import inputs

pytestmark = pytest.mark.gpu


def test_windowed_error_is_small_and_below_naive():
    wl = inputs.Workload("gdn_outlier_b4_h8_d128_w64", 4, 8, 128, 128, 64, 2, 2, False, 0, 320,
                         torch.bfloat16, 3, planted=True)
    r = bench.quality(wl, torch.device("cuda", 0))
    win, naive = r["per_window"]["windowed"], r["per_window"]["naive"]
    assert len(win) == 5 and all(x == x for x in win + naive)
    assert r["rel_l2_windowed_vs_fp32"] < 1e-2, r
    assert r["naive_over_windowed"] > 5.0, r
    assert all(w < n for w, n in zip(win, naive)), r
