"""Checkpoint and resume: a state copied mid-window into a new handle continues
exactly as the original (outputs and encoded state bit for bit)."""
import numpy as np
import pytest
import torch

from harness import to_device
from recurrent_state_quantization_lq_b200 import inputs, lq

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _continue(st, tb, t0, t1, W, masks=None):
    outs = []
    for t in range(t0, t1):
        act = None if masks is None else torch.tensor(masks[t].astype(np.uint8), device=DEV)
        o = st.decode_step(tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t], active=act)
        if act is not None:                  # rows of inactive sequences are not written
            o = torch.where(act.bool()[:, None, None], o, torch.zeros((), device=DEV))
        outs.append(o.clone())
        if st.ragged:
            st.flush()
        elif st.fill == W:
            st.flush()
    return torch.stack(outs)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_resume_mid_window_shared_phase(gate):
    d, B, H, W, T1, T2 = 128, 2, 3, 8, 11, 14
    tb = to_device(inputs.tokens(51, 0, T1 + T2, B, H, d, d, gate == "channel"), DEV)
    S0 = (0.5 * torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(51))).to(DEV)
    a = lq.DecodeState(B, H, d, window=W, gate=gate, device=DEV)
    a.prefill(S0)
    _continue(a, tb, 0, T1, W)
    ws, n = a.checkpoint()
    assert n == T1 % W
    b = lq.DecodeState(B, H, d, window=W, gate=gate, device=DEV)    # another workspace address
    b.resume(ws, n)
    oa = _continue(a, tb, T1, T1 + T2, W)
    ob = _continue(b, tb, T1, T1 + T2, W)
    assert torch.equal(oa, ob)
    assert torch.equal(a.workspace, b.workspace)
    assert a.device_status() == lq.LQ_OK and b.device_status() == lq.LQ_OK


def test_resume_ragged_phases():
    d, B, H, W, T1, T2 = 64, 4, 2, 5, 9, 12
    tb = to_device(inputs.tokens(52, 0, T1 + T2, B, H, d, d, False), DEV)
    masks = np.random.default_rng(52).random((T1 + T2, B)) < 0.7
    a = lq.DecodeState(B, H, d, window=W, ragged=True, device=DEV)
    a.prefill(None)
    _continue(a, tb, 0, T1, W, masks)
    ws, n = a.checkpoint()
    b = lq.DecodeState(B, H, d, window=W, ragged=True, device=DEV)
    b.resume(ws, n)
    assert torch.equal(a.fills(), b.fills())
    oa = _continue(a, tb, T1, T1 + T2, W, masks)
    ob = _continue(b, tb, T1, T1 + T2, W, masks)
    assert torch.equal(oa, ob)
    assert torch.equal(a.workspace, b.workspace)
