"""Parity at the full benchmark sizes, in the launch configuration the
benchmark times (one launch per decode step over every (sequence, head)).

The oracle recomputes a seeded sample of (sequence, head) units one by one:
its own FP64 prefill from the zero state, then the windowed decode.  The
whole output tensor is also checked for properties that hold at any size.
"""
import numpy as np
import pytest
import torch

import oracle
from recurrent_state_quantization_lq_b200 import inputs, lq

from harness import compare_codes, gpu_run, import_encoded, oracle_params, rel_l2, to_device, unit_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(wl: inputs.Workload, decode_tokens: int, n_sample: int):
    B, H, d, W = wl.batch, wl.heads, wl.d_k, wl.window
    gate = "channel" if wl.per_channel_gate else "scalar"
    P = wl.prefill_tokens
    tb_pre = inputs.tokens(wl.seed, 0, P, B, H, d, d, wl.per_channel_gate, wl.dtype)
    tb_dec = inputs.tokens(wl.seed, P, P + decode_tokens, B, H, d, d, wl.per_channel_gate, wl.dtype)

    # GPU: FP32 prefill from zero, then the windowed INT8 decode
    pre = lq.DecodeState(B, H, d, gate=gate, mode="fp32", in_dtype=wl.dtype, device=DEV)
    pre.prefill(None)
    gpu_run(pre, to_device(tb_pre, DEV))
    S0 = pre.view("state_f32").clone()
    st = lq.DecodeState(B, H, d, window=W, n_comp_rows=wl.n_comp_rows, n_comp_cols=wl.n_comp_cols,
                        gate=gate, in_dtype=wl.dtype, device=DEV)
    st.prefill(S0)
    first_codes = st.view("codes").cpu().clone()
    tbd = to_device(tb_dec, DEV)
    o_gpu, shots = gpu_run(st, tbd, flush_every=W)
    assert st.device_status() == lq.LQ_OK

    # properties of the whole output and state
    assert torch.isfinite(o_gpu).all()
    for snap in shots:
        c = snap["codes"].reshape(B * H, d, d)
        assert c.abs().max() <= 127
        live = snap["row_scale"].reshape(B * H, d) > 0
        assert (c.abs().amax(dim=2)[live] == 127).all()

    # the oracle on a seeded sample of units
    rng = np.random.default_rng(wl.seed)
    units = sorted(rng.choice(B * H, n_sample, replace=False).tolist())
    zeros = np.zeros((n_sample, d, d))
    ref_pre = oracle.run(oracle_params(d, gate=gate, mode="fp32"), zeros, *unit_inputs(tb_pre, units))
    S0_gpu = S0.reshape(B * H, d, d)[units].cpu().numpy()
    assert rel_l2(S0_gpu, ref_pre.S_final) <= 1e-5
    p = oracle_params(d, W, wl.n_comp_rows, wl.n_comp_cols, gate)
    ref = oracle.run(p, ref_pre.S_final, *unit_inputs(tb_dec, units))

    o_s = o_gpu.reshape(decode_tokens, B * H, d)[:, units].transpose(0, 1).numpy()
    err = rel_l2(o_s, ref.o)
    assert err <= 1e-3, err
    # codes of the prefill encoding and of the first flush (no cascade before it)
    for f, c in enumerate([first_codes, shots[0]["codes"]]):
        frac, worst = compare_codes(c.reshape(B * H, d, d)[units].numpy(), ref.Q[:, f])
        assert frac >= 0.999 and worst <= 1, (f, frac, worst)

    # teacher-forced window: the sampled units restart from the oracle's encoding
    st.prefill(S0)
    import_encoded(st, ref, 0, units)
    o_w, snaps = gpu_run(st, inputs.TokenBatch(*(x[:W] for x in (tbd.q, tbd.k, tbd.v, tbd.g, tbd.beta))),
                         flush_every=W)
    o_ws = o_w.reshape(W, B * H, d)[:, units].transpose(0, 1).numpy()
    assert rel_l2(o_ws, ref.o[:, :W]) <= 1e-5
    c = snaps[0]["codes"].reshape(B * H, d, d)[units].numpy()
    idx = snaps[0]["comp_index"].reshape(B * H, -1)[units].numpy()[:, :wl.n_comp_rows + wl.n_comp_cols]
    keep = (idx == ref.idx[:, 1]).all(axis=1)
    assert keep.sum() >= len(units) - 1
    frac, worst = compare_codes(c[keep], ref.Q[keep, 1])
    assert frac >= 0.999 and worst <= 1, (frac, worst)
    return err


def test_gdn_b64_h32_d128_w64_sampled():
    wl = inputs.WORKLOADS["gdn_b64_h32_d128_w64"]
    _run(wl, decode_tokens=2 * wl.window, n_sample=8)


def test_kda_b128_h32_d128_w128_sampled():
    wl = inputs.WORKLOADS["kda_b128_h32_d128_w128"]
    _run(wl, decode_tokens=wl.window + 32, n_sample=6)
