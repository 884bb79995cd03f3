"""Parity at the full benchmark sizes, in the launch configuration the
benchmark times (one launch per decode step over every (sequence, head)).

The oracle recomputes a seeded sample of (sequence, head) units one by one:
its own FP64 prefill from the zero state (or the same planted state), then the
windowed decode.  Free-running outputs are compared over the whole run, and
every window is also run teacher-forced: the sampled units restart from the
oracle's encoding of that window, and their outputs and flushed codes are
compared with the oracle's.  The whole output tensor and every flushed state
are also checked for properties that hold at any size.
"""
import numpy as np
import pytest
import torch

import oracle
from recurrent_state_quantization_lq_b200 import inputs, lq

from harness import (compare_codes, decoded_state, gpu_run, import_encoded, oracle_params, rel_l2,
                     selection_is_near_tie, to_device, unit_inputs)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _sampled_case(B, H, d, W, nr, nc, gate, dtype, seed, n_windows, n_sample, prefill_tokens=0,
                  S0=None, extra_tokens=0):
    """Windowed decode of B x H units over n_windows windows (+ extra tokens),
    from S0 (CPU FP32 [B, H, d, d]) or from the FP32 recurrence over
    prefill_tokens tokens from zero, checked on n_sample seeded units."""
    per_ch = gate == "channel"
    P = prefill_tokens
    T = n_windows * W + extra_tokens
    tb_dec = inputs.tokens(seed, P, P + T, B, H, d, d, per_ch, dtype)
    if S0 is None:
        tb_pre = inputs.tokens(seed, 0, P, B, H, d, d, per_ch, dtype)
        pre = lq.DecodeState(B, H, d, gate=gate, mode="fp32", in_dtype=dtype, device=DEV)
        pre.prefill(None)
        gpu_run(pre, to_device(tb_pre, DEV))
        S0_dev = pre.read("state_f32", device=DEV)
        del pre
    else:
        S0_dev = S0.to(DEV).contiguous()
    st = lq.DecodeState(B, H, d, window=W, n_comp_rows=nr, n_comp_cols=nc, gate=gate, in_dtype=dtype,
                        device=DEV)
    st.prefill(S0_dev)
    first_codes = st.read("codes")
    tbd = to_device(tb_dec, DEV)
    o_gpu, shots = gpu_run(st, tbd, flush_every=W)
    assert st.device_status() == lq.LQ_OK

    # properties of the whole output and of every flushed state
    assert torch.isfinite(o_gpu).all()
    for snap in shots:
        c = snap["codes"].reshape(B * H, d, d)
        assert c.abs().max() <= 127
        live = snap["row_scale"].reshape(B * H, d) > 0
        assert (c.abs().amax(dim=2)[live] == 127).all()
        assert (snap["col_smooth"] > 0).all()
        if nr + nc:
            idx = snap["comp_index"].reshape(B * H, nr + nc)
            assert ((idx >= 0) & (idx < d)).all()
            rows, cols = idx[:, :nr].sort(dim=1).values, idx[:, nr:].sort(dim=1).values
            assert (rows[:, 1:] != rows[:, :-1]).all() and (cols[:, 1:] != cols[:, :-1]).all()

    # the oracle on a seeded sample of units
    rng = np.random.default_rng(seed)
    units = sorted(rng.choice(B * H, n_sample, replace=False).tolist())
    if S0 is None:
        zeros = np.zeros((n_sample, d, d))
        ref_pre = oracle.run(oracle_params(d, gate=gate, mode="fp32"), zeros, *unit_inputs(tb_pre, units),
                             snapshots=False)
        S0_gpu = S0_dev.reshape(B * H, d, d)[units].cpu().numpy()
        assert rel_l2(S0_gpu, ref_pre.S_final) <= 1e-5
        S0_ref = ref_pre.S_final
    else:
        S0_ref = S0.reshape(B * H, d, d)[units].double().numpy()
    p = oracle_params(d, W, nr, nc, gate)
    q, k, v, g, beta = unit_inputs(tb_dec, units)
    ref = oracle.run(p, S0_ref, q, k, v, g, beta)

    o_s = o_gpu.reshape(T, B * H, d)[:, units].transpose(0, 1).numpy()
    err = rel_l2(o_s, ref.o)
    assert err <= 1e-3, err
    # codes of the prefill encoding and of the first flush (no cascade before it)
    for f, c in enumerate([first_codes, shots[0]["codes"]]):
        frac, worst = compare_codes(c.reshape(B * H, d, d)[units].numpy(), ref.Q[:, f])
        assert frac >= 0.999 and worst <= 1, (f, frac, worst)

    # teacher-forced windows: the sampled units restart from the oracle's encoding
    plain = oracle_params(d, gate=gate, mode="fp32")
    for w in range(n_windows):
        st.prefill(S0_dev)
        import_encoded(st, ref, w, units)
        sl = slice(w * W, (w + 1) * W)
        o_w, snaps = gpu_run(st, inputs.TokenBatch(*(x[sl] for x in (tbd.q, tbd.k, tbd.v, tbd.g, tbd.beta))),
                             flush_every=W)
        assert st.device_status() == lq.LQ_OK
        o_ws = o_w.reshape(W, B * H, d)[:, units].transpose(0, 1).numpy()
        e_w = rel_l2(o_ws, ref.o[:, sl])
        assert e_w <= 1e-5, ("teacher-forced outputs", w, e_w)
        c = snaps[0]["codes"].reshape(B * H, d, d)[units].numpy()
        keep = np.ones(n_sample, bool)
        if nr + nc:
            got_idx = snaps[0]["comp_index"].reshape(B * H, nr + nc)[units].numpy()
            flips = np.nonzero((got_idx != ref.idx[:, w + 1]).any(axis=1))[0]
            if len(flips):
                S_tilde = decoded_state(ref, w, nr, nc, d)
                pre_flush = oracle.run(plain, S_tilde[flips], q[flips, sl], k[flips, sl], v[flips, sl],
                                       g[flips, sl], beta[flips, sl], snapshots=False).S_final
                for i, n in enumerate(flips):
                    assert selection_is_near_tie(pre_flush[i], got_idx[n], ref.idx[n, w + 1], nr), (w, n)
                keep[flips] = False
        frac, worst = compare_codes(c[keep], ref.Q[keep, w + 1])
        assert frac >= 0.999 and worst <= 1, ("teacher-forced flush", w, frac, worst)
    return err


def test_gdn_b64_h32_d128_w64_sampled():
    """The benchmark's workload: 64 sampled units, four windows after a 512-token prefill."""
    wl = inputs.WORKLOADS["gdn_b64_h32_d128_w64"]
    _sampled_case(wl.batch, wl.heads, wl.d_k, wl.window, wl.n_comp_rows, wl.n_comp_cols, "scalar", wl.dtype,
                  wl.seed, n_windows=4, n_sample=64, prefill_tokens=wl.prefill_tokens)


def test_kda_b128_h32_d128_w128_sampled():
    """Per-key-channel gate, W = 128, 4 + 4 compensators: 64 sampled units, four windows."""
    wl = inputs.WORKLOADS["kda_b128_h32_d128_w128"]
    _sampled_case(wl.batch, wl.heads, wl.d_k, wl.window, wl.n_comp_rows, wl.n_comp_cols, "channel", wl.dtype,
                  wl.seed, n_windows=4, n_sample=64, prefill_tokens=wl.prefill_tokens)


def test_gdn_outlier_planted_sampled():
    """The outlier-stress recipe (2 rows and 2 columns planted x 50 over an N(0, 1)
    state, W = 64, 2 + 2 compensators) at 32 sequences x 32 heads, four windows,
    against the oracle on 32 sampled units."""
    wl = inputs.WORKLOADS["gdn_outlier_b256_h32_d128_w64"]
    B = 32
    S0 = inputs.planted_state(wl.seed, B, wl.heads, wl.d_v, wl.d_k)[0]
    _sampled_case(B, wl.heads, wl.d_k, wl.window, wl.n_comp_rows, wl.n_comp_cols, "scalar", wl.dtype, wl.seed,
                  n_windows=4, n_sample=32, S0=S0)


def test_gdn_sweep_b512_w256_sampled():
    """The sweep's largest point (512 sequences x 32 heads, W = 256), where every
    CTA walks many units: one full window plus 8 tokens, 16 sampled units."""
    wl = inputs.sweep_workload(512, 256)
    S0 = 0.5 * torch.randn(wl.batch, wl.heads, wl.d_v, wl.d_k, generator=torch.Generator().manual_seed(wl.seed))
    _sampled_case(wl.batch, wl.heads, wl.d_k, wl.window, wl.n_comp_rows, wl.n_comp_cols, "scalar", wl.dtype,
                  wl.seed, n_windows=1, n_sample=16, S0=S0, extra_tokens=8)
