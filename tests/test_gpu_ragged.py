"""Ragged window phases on the GPU against the oracle.

Each sequence of a ragged state keeps its own window: per step only the active
sequences take a token, every unit whose window holds W tokens is flushed, and
a batch slot can be restarted from a new state mid-stream.  The reference for
one (sequence, head) unit is the oracle run over that unit's own tokens (its
active steps), with a window of W of its tokens - the windowed scheme of
LeapQuant ("LeapQuant: Efficient Linear Attention with Accurate Recurrent State
Quantization", section "Abstract (arXiv)") applied per sequence.
"""
import numpy as np
import pytest
import torch

import oracle
from harness import oracle_params, rel_l2, to_device, unit_inputs
from recurrent_state_quantization_lq_b200 import inputs, lq

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _ragged_case(d, gate, dtype, W, nr, nc, B, H, T, seed, join_at=None, p_active=0.7):
    per_channel = gate == "channel"
    tb = inputs.tokens(seed, 0, T, B, H, d, d, per_channel, dtype)
    rng = np.random.default_rng(seed)
    active = rng.random((T, B)) < p_active
    gen = torch.Generator().manual_seed(seed)
    S0 = 0.5 * torch.randn(B, H, d, d, generator=gen)
    S1 = 0.5 * torch.randn(B, H, d, d, generator=gen)          # the state a joining sequence starts from
    join_seq = 1 % B

    st = lq.DecodeState(B, H, d, window=W, n_comp_rows=nr, n_comp_cols=nc, gate=gate, in_dtype=dtype,
                        ragged=True, device=DEV)
    st.prefill(S0.to(DEV).contiguous())
    tbd = to_device(tb, DEV)
    out = torch.full((T, B, H, d), float("nan"), device=DEV)
    mask = torch.zeros(B, dtype=torch.uint8, device=DEV)
    mask[join_seq] = 1
    for t in range(T):
        if join_at is not None and t == join_at:
            st.prefill_sequences(S1.to(DEV).contiguous(), mask)
        act = torch.tensor(active[t].astype(np.uint8), device=DEV)
        st.decode_step(tbd.q[t], tbd.k[t], tbd.v[t], tbd.g[t], tbd.beta[t], out=out[t], active=act)
        st.flush()
    assert st.device_status() == lq.LQ_OK, lq.last_error()
    fills = st.fills().cpu().numpy()
    o_gpu = out.cpu().numpy()

    p = oracle_params(d, W, nr, nc, gate, "window")
    q, k, v, g, beta = unit_inputs(tb, range(B * H))
    got, ref = [], []
    for b in range(B):
        for h in range(H):
            u = b * H + h
            steps = np.nonzero(active[:, b])[0]
            segments = [(S0[b, h], steps)]
            if join_at is not None and b == join_seq:
                segments = [(S0[b, h], steps[steps < join_at]), (S1[b, h], steps[steps >= join_at])]
            for S_start, seg in segments:
                if len(seg) == 0:
                    continue
                r = oracle.run(p, S_start.double().numpy()[None], q[u:u + 1, seg], k[u:u + 1, seg],
                               v[u:u + 1, seg], g[u:u + 1, seg], beta[u:u + 1, seg], snapshots=False)
                ref.append(r.o[0])
                got.append(o_gpu[seg, b, h])
            last = segments[-1][1]
            assert fills[b, h] == len(last) % W, (b, h, fills[b, h], len(last))
            # inactive steps leave the output rows untouched
            idle = np.setdiff1d(np.arange(T), steps)
            assert np.isnan(o_gpu[idle, b, h]).all()
    err = rel_l2(np.concatenate(got), np.concatenate(ref))
    assert err <= 1e-3, err
    st.flush_pending()
    assert st.device_status() == lq.LQ_OK
    assert int(st.fills().abs().sum()) == 0
    return err


@pytest.mark.parametrize("d,gate,dtype", [(64, "scalar", torch.bfloat16), (128, "scalar", torch.bfloat16),
                                          (128, "channel", torch.bfloat16), (64, "scalar", torch.float32)])
def test_ragged_phases_match_per_sequence_oracle(d, gate, dtype):
    _ragged_case(d, gate, dtype, W=8, nr=2, nc=2, B=3, H=2, T=40, seed=31)


def test_ragged_join_restarts_one_sequence():
    _ragged_case(128, "scalar", torch.bfloat16, W=6, nr=1, nc=1, B=4, H=2, T=30, seed=7, join_at=13)


def test_ragged_decode_into_full_window_is_reported():
    d, B, H, W = 64, 2, 2, 4
    tb = to_device(inputs.tokens(3, 0, W + 1, B, H, d, d, False), DEV)
    st = lq.DecodeState(B, H, d, window=W, ragged=True, device=DEV)
    st.prefill(None)
    for t in range(W + 1):                      # no flush: the last step finds full windows
        st.decode_step(tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t])
    assert st.device_status() == lq.LQ_ERR_WINDOW_FULL
    assert (st.fills() == W).all()
    st.flush()                                  # full windows are flushed
    assert (st.fills() == 0).all()
    st.prefill(None)                            # prefill clears the error word
    assert st.device_status() == lq.LQ_OK
