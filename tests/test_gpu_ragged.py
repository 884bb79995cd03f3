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


def _ragged_case(d, gate, dtype, W, nr, nc, B, H, T, seed, join_at=None, p_active=0.7, sample=None,
                 zero_start=False):
    per_channel = gate == "channel"
    tb = inputs.tokens(seed, 0, T, B, H, d, d, per_channel, dtype)
    rng = np.random.default_rng(seed)
    active = rng.random((T, B)) < p_active
    if zero_start:
        S0 = S1 = None
    else:
        gen = torch.Generator().manual_seed(seed)
        S0 = 0.5 * torch.randn(B, H, d, d, generator=gen)
        S1 = 0.5 * torch.randn(B, H, d, d, generator=gen)      # the state a joining sequence starts from
    join_seq = 1 % B

    st = lq.DecodeState(B, H, d, window=W, n_comp_rows=nr, n_comp_cols=nc, gate=gate, in_dtype=dtype,
                        ragged=True, device=DEV)
    st.prefill(None if zero_start else S0.to(DEV).contiguous())
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
    # every unit's count: its tokens since it last held W (or since its restart)
    expect = np.zeros(B, dtype=np.int64)
    for t in range(T):
        if join_at is not None and t == join_at:
            expect[join_seq] = 0
        expect = np.where(active[t], (expect + 1) % W, expect)
    assert (fills == expect[:, None]).all()

    p = oracle_params(d, W, nr, nc, gate, "window")
    pairs = [(b, h) for b in range(B) for h in range(H)] if sample is None else sample
    q, k, v, g, beta = unit_inputs(tb, [b * H + h for b, h in pairs])
    got, ref = [], []
    for u, (b, h) in enumerate(pairs):
        steps = np.nonzero(active[:, b])[0]
        start = np.zeros((d, d)) if zero_start else S0[b, h].double().numpy()
        segments = [(start, steps)]
        if join_at is not None and b == join_seq:
            segments = [(start, steps[steps < join_at]), (S1[b, h].double().numpy(), steps[steps >= join_at])]
        for S_start, seg in segments:
            if len(seg) == 0:
                continue
            r = oracle.run(p, S_start[None], q[u:u + 1, seg], k[u:u + 1, seg], v[u:u + 1, seg], g[u:u + 1, seg],
                           beta[u:u + 1, seg], snapshots=False)
            ref.append(r.o[0])
            got.append(o_gpu[seg, b, h])
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
                                          (128, "channel", torch.bfloat16), (64, "scalar", torch.float32),
                                          (64, "channel", torch.bfloat16), (128, "scalar", torch.float32),
                                          (128, "channel", torch.float32), (64, "channel", torch.float32)])
def test_ragged_phases_match_per_sequence_oracle(d, gate, dtype):
    _ragged_case(d, gate, dtype, W=8, nr=2, nc=2, B=3, H=2, T=40, seed=31)


def test_ragged_max_select_and_no_compensators():
    _ragged_case(128, "scalar", torch.bfloat16, W=5, nr=0, nc=0, B=2, H=3, T=17, seed=12)
    _ragged_case(128, "scalar", torch.bfloat16, W=40, nr=8, nc=8, B=2, H=2, T=90, seed=13, p_active=0.9)


def test_ragged_many_units_scan_in_passes():
    """65,536 units: each persistent cluster scans its candidates in more than
    one pass of 128; the oracle checks a sample of units."""
    B, H = 2048, 32
    rng = np.random.default_rng(5)
    sample = [(int(b), int(h)) for b, h in zip(rng.integers(0, B, 48), rng.integers(0, H, 48))]
    sample += [(0, 0), (B - 1, H - 1), (B // 2, 7)]
    _ragged_case(64, "scalar", torch.bfloat16, W=4, nr=1, nc=1, B=B, H=H, T=9, seed=17, sample=sample,
                 zero_start=True)


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


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_ragged_without_masks_matches_shared_phase(gate):
    """No active mask: every unit keeps the same phase, and a ragged handle
    flushed after every step gives exactly the shared-phase handle's outputs
    and encoded state."""
    d, B, H, W, T = 128, 3, 2, 8, 21
    tb = to_device(inputs.tokens(41, 0, T, B, H, d, d, gate == "channel"), DEV)
    S0 = (0.5 * torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(41))).to(DEV)
    rag = lq.DecodeState(B, H, d, window=W, gate=gate, ragged=True, device=DEV)
    ref = lq.DecodeState(B, H, d, window=W, gate=gate, device=DEV)
    rag.prefill(S0)
    ref.prefill(S0)
    o_rag = torch.empty(T, B, H, d, device=DEV)
    o_ref = torch.empty(T, B, H, d, device=DEV)
    for t in range(T):
        rag.decode_step(tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t], out=o_rag[t])
        rag.flush()
        ref.decode_step(tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t], out=o_ref[t])
        if ref.fill == W:
            ref.flush()
    assert rag.device_status() == lq.LQ_OK and ref.device_status() == lq.LQ_OK
    assert torch.equal(o_rag, o_ref)
    for name in ("codes", "row_scale", "col_smooth", "comp_index", "buf_delta"):
        assert torch.equal(rag.read(name), ref.read(name)), name
    assert (rag.fills() == T % W).all()


def test_ragged_phases_realign_after_flush_pending():
    """Masked steps, then a pending flush (every partial window encoded), then
    unmasked steps: each unit follows the oracle run over its own tokens, its
    partial window ending at the pending flush."""
    d, B, H, W, T1, T2 = 64, 4, 2, 6, 13, 11
    T = T1 + T2
    tb = inputs.tokens(23, 0, T, B, H, d, d, False)
    rng = np.random.default_rng(23)
    active = np.ones((T, B), dtype=bool)
    active[:T1] = rng.random((T1, B)) < 0.6
    S0 = 0.5 * torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(23))
    st = lq.DecodeState(B, H, d, window=W, n_comp_rows=1, n_comp_cols=1, ragged=True, device=DEV)
    st.prefill(S0.to(DEV))
    tbd = to_device(tb, DEV)
    out = torch.full((T, B, H, d), float("nan"), device=DEV)
    for t in range(T):
        if t == T1:
            st.flush_pending()
        if t < T1:
            act = torch.tensor(active[t].astype(np.uint8), device=DEV)
            st.decode_step(tbd.q[t], tbd.k[t], tbd.v[t], tbd.g[t], tbd.beta[t], out=out[t], active=act)
        else:
            st.decode_step(tbd.q[t], tbd.k[t], tbd.v[t], tbd.g[t], tbd.beta[t], out=out[t])
        st.flush()
    assert st.device_status() == lq.LQ_OK, lq.last_error()
    assert (st.fills() == T2 % W).all()
    o_gpu = out.cpu().numpy()
    p = oracle_params(d, W, 1, 1, "scalar", "window")
    q, k, v, g, beta = unit_inputs(tb, range(B * H))
    got, ref = [], []
    for b in range(B):
        for h in range(H):
            u = b * H + h
            s1 = np.nonzero(active[:T1, b])[0]
            s2 = np.arange(T1, T)
            S_start = S0[b, h].double().numpy()[None]
            if len(s1):
                r1 = oracle.run(p, S_start, q[u:u + 1, s1], k[u:u + 1, s1], v[u:u + 1, s1], g[u:u + 1, s1],
                                beta[u:u + 1, s1], snapshots=False)
                ref.append(r1.o[0])
                got.append(o_gpu[s1, b, h])
                S_start = r1.S_final          # the pending flush encodes the window where it stands
            r2 = oracle.run(p, S_start, q[u:u + 1, s2], k[u:u + 1, s2], v[u:u + 1, s2], g[u:u + 1, s2],
                            beta[u:u + 1, s2], snapshots=False)
            ref.append(r2.o[0])
            got.append(o_gpu[s2, b, h])
    err = rel_l2(np.concatenate(got), np.concatenate(ref))
    assert err <= 1e-3, err


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_ragged_restart_from_prompts_of_different_lengths(gate):
    """Sequences 1 and 3 restart mid-stream from their own prompts (lengths 5
    and 0 of a 7-token padded batch); each restarted unit follows the oracle's
    FP32 recurrence over its prompt, the encoded result, then the windowed run
    over its later tokens.  The other sequences are untouched."""
    d, B, H, W, T, J, P = 64, 4, 2, 5, 18, 9, 7
    lengths = np.array([7, 5, 3, 0], dtype=np.int32)
    mask = np.array([0, 1, 0, 1], dtype=np.uint8)
    per_channel = gate == "channel"
    tb = inputs.tokens(71, 0, T, B, H, d, d, per_channel)
    pb = inputs.tokens(72, 0, P, B, H, d, d, per_channel)
    rng = np.random.default_rng(71)
    active = rng.random((T, B)) < 0.75
    gen = torch.Generator().manual_seed(71)
    S0 = 0.5 * torch.randn(B, H, d, d, generator=gen)
    S1 = 0.5 * torch.randn(B, H, d, d, generator=gen)
    st = lq.DecodeState(B, H, d, window=W, n_comp_rows=1, n_comp_cols=1, gate=gate, ragged=True, device=DEV)
    st.prefill(S0.to(DEV).contiguous())
    tbd, pbd = to_device(tb, DEV), to_device(pb, DEV)
    out = torch.full((T, B, H, d), float("nan"), device=DEV)
    pout = torch.full((P, B, H, d), float("nan"), device=DEV)
    for t in range(T):
        if t == J:
            st.prefill_sequences_tokens(pbd.q, pbd.k, pbd.v, pbd.g, pbd.beta,
                                        torch.tensor(mask, device=DEV), torch.tensor(lengths, device=DEV),
                                        S0=S1.to(DEV).contiguous(), out=pout)
        act = torch.tensor(active[t].astype(np.uint8), device=DEV)
        st.decode_step(tbd.q[t], tbd.k[t], tbd.v[t], tbd.g[t], tbd.beta[t], out=out[t], active=act)
        st.flush()
    assert st.device_status() == lq.LQ_OK, lq.last_error()
    o_gpu, p_gpu = out.cpu().numpy(), pout.cpu().numpy()
    pw = oracle_params(d, W, 1, 1, gate, "window")
    pf = oracle_params(d, W, 1, 1, gate, "fp32")
    q, k, v, g, beta = unit_inputs(tb, range(B * H))
    pq, pk, pv, pg, pbeta = unit_inputs(pb, range(B * H))
    got, ref, pgot, pref = [], [], [], []
    for b in range(B):
        for h in range(H):
            u = b * H + h
            steps = np.nonzero(active[:, b])[0]
            segs = [(S0[b, h].double().numpy()[None], steps)]
            if mask[b]:
                L = int(lengths[b])
                S_start = S1[b, h].double().numpy()[None]
                if L:
                    rp = oracle.run(pf, S_start, pq[u:u + 1, :L], pk[u:u + 1, :L], pv[u:u + 1, :L],
                                    pg[u:u + 1, :L], pbeta[u:u + 1, :L], snapshots=False)
                    pref.append(rp.o[0])
                    pgot.append(p_gpu[:L, b, h])
                    S_start = rp.S_final
                assert np.isnan(p_gpu[L:, b, h]).all()
                segs = [(segs[0][0], steps[steps < J]), (S_start, steps[steps >= J])]
            else:
                assert np.isnan(p_gpu[:, b, h]).all()
            for S_s, seg in segs:
                if len(seg) == 0:
                    continue
                r = oracle.run(pw, S_s, q[u:u + 1, seg], k[u:u + 1, seg], v[u:u + 1, seg], g[u:u + 1, seg],
                               beta[u:u + 1, seg], snapshots=False)
                ref.append(r.o[0])
                got.append(o_gpu[seg, b, h])
    assert rel_l2(np.concatenate(pgot), np.concatenate(pref)) <= 1e-5
    err = rel_l2(np.concatenate(got), np.concatenate(ref))
    assert err <= 1e-3, err


@pytest.mark.parametrize("seed", [101, 202])
def test_ragged_random_operation_mix(seed):
    """Random masked decodes with a flush after each step, interleaved with
    sequence restarts from a state or from a prompt and with pending flushes.
    Each unit's outputs follow the oracle over its own segments: a restart
    starts a segment from its new state (after the prompt's FP32 recurrence);
    a pending flush ends the unit's partial window, so its next segment starts
    from the oracle's state at that token."""
    d, B, H, W, T, P = 64, 4, 2, 5, 36, 6
    rng = np.random.default_rng(seed)
    tb = inputs.tokens(seed, 0, T, B, H, d, d, False)
    pb = inputs.tokens(seed + 1, 0, P, B, H, d, d, False)
    gen = torch.Generator().manual_seed(seed)
    S0 = 0.5 * torch.randn(B, H, d, d, generator=gen)
    S1 = 0.5 * torch.randn(B, H, d, d, generator=gen)
    st = lq.DecodeState(B, H, d, window=W, n_comp_rows=1, n_comp_cols=1, ragged=True, device=DEV)
    st.prefill(S0.to(DEV).contiguous())
    tbd, pbd = to_device(tb, DEV), to_device(pb, DEV)
    out = torch.full((T, B, H, d), float("nan"), device=DEV)
    pout = torch.full((P, B, H, d), float("nan"), device=DEV)
    # per sequence: a list of segments (kind, start info, token steps)
    segs = [[["state", "S0", []]] for _ in range(B)]
    fill = np.zeros(B, dtype=np.int64)
    prompt_used = False
    events = {"state": 0, "prompt": 0, "pending": 0}
    for t in range(T):
        event = rng.random()
        if event < 0.08 and t > 0:                                   # restart sequences from a state
            mask = (rng.random(B) < 0.5).astype(np.uint8)
            st.prefill_sequences(S1.to(DEV).contiguous(), torch.tensor(mask, device=DEV))
            events["state"] += 1
            for b in np.nonzero(mask)[0]:
                segs[b].append(["state", "S1", []])
                fill[b] = 0
        elif event < 0.14 and t > 0 and not prompt_used:            # restart from prompts
            mask = (rng.random(B) < 0.5).astype(np.uint8)
            lengths = rng.integers(0, P + 1, B).astype(np.int32)
            st.prefill_sequences_tokens(pbd.q, pbd.k, pbd.v, pbd.g, pbd.beta, torch.tensor(mask, device=DEV),
                                        torch.tensor(lengths, device=DEV), S0=S1.to(DEV).contiguous(), out=pout)
            prompt_used = True
            events["prompt"] += 1
            for b in np.nonzero(mask)[0]:
                segs[b].append(["prompt", int(lengths[b]), []])
                fill[b] = 0
        elif event < 0.2 and t > 0:                                  # end every partial window
            st.flush_pending()
            events["pending"] += 1
            for b in range(B):
                if fill[b] > 0:
                    segs[b].append(["continue", None, []])
                fill[b] = 0
        act = rng.random(B) < 0.7
        st.decode_step(tbd.q[t], tbd.k[t], tbd.v[t], tbd.g[t], tbd.beta[t], out=out[t],
                       active=torch.tensor(act.astype(np.uint8), device=DEV))
        st.flush()
        for b in np.nonzero(act)[0]:
            segs[b][-1][2].append(t)
            fill[b] = (fill[b] + 1) % W
    assert min(events.values()) >= 1, events          # the seed exercises every operation
    assert st.device_status() == lq.LQ_OK, lq.last_error()
    assert (st.fills().cpu().numpy() == fill[:, None]).all()
    o_gpu, p_gpu = out.cpu().numpy(), pout.cpu().numpy()
    pw = oracle_params(d, W, 1, 1, "scalar", "window")
    pf = oracle_params(d, W, 1, 1, "scalar", "fp32")
    q, k, v, g, beta = unit_inputs(tb, range(B * H))
    pq, pk, pv, pg, pbeta = unit_inputs(pb, range(B * H))
    got, ref = [], []
    for b in range(B):
        for h in range(H):
            u = b * H + h
            S = None
            for kind, info, steps in segs[b]:
                if kind == "state":
                    S = (S0 if info == "S0" else S1)[b, h].double().numpy()[None]
                elif kind == "prompt":
                    S = S1[b, h].double().numpy()[None]
                    if info:
                        rp = oracle.run(pf, S, pq[u:u + 1, :info], pk[u:u + 1, :info], pv[u:u + 1, :info],
                                        pg[u:u + 1, :info], pbeta[u:u + 1, :info], snapshots=False)
                        got.append(p_gpu[:info, b, h])
                        ref.append(rp.o[0])
                        S = rp.S_final
                if not steps:
                    continue
                s = np.array(steps)
                r = oracle.run(pw, S, q[u:u + 1, s], k[u:u + 1, s], v[u:u + 1, s], g[u:u + 1, s],
                               beta[u:u + 1, s], snapshots=False)
                got.append(o_gpu[s, b, h])
                ref.append(r.o[0])
                S = r.S_final                 # a later "continue" segment starts here
    err = rel_l2(np.concatenate(got), np.concatenate(ref))
    assert err <= 1e-3, err
