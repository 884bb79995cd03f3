"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Tolerances:
  * codec on a given FP32 state (prefill): bit-exact codes, row scales,
    smoothing factors, compensator indices and vectors; both sides take every
    decision in IEEE FP32 with correctly rounded division and square root.
  * decode outputs: relative L2 error <= 1e-3 over the whole output tensor
    (the method's stated bar); the FP32-state comparator <= 1e-5.
  * codes after a window flush: >= 99.9 % equal and never more than 1 LSB
    apart (the rebuilt FP32 state differs from the FP64 oracle's by rounding,
    which moves a code only where it sits on a rounding boundary).
"""
import numpy as np
import pytest
import torch

import oracle
from recurrent_state_quantization_lq_b200 import inputs, lq

from harness import (compare_codes, decoded_state, gpu_run, import_encoded, oracle_params, rel_l2,
                     selection_is_near_tie, snapshot, to_device, unit_inputs)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _state(kind, seed, B, H, d):
    g = torch.Generator().manual_seed(seed)
    if kind == "zero":
        return torch.zeros(B, H, d, d)
    if kind == "planted":
        return inputs.planted_state(seed, B, H, d, d)[0]
    S = torch.randn(B, H, d, d, generator=g)
    if kind == "scaled":   # rows spanning six orders of magnitude, some exactly zero
        S = S * torch.logspace(-3, 3, d)[torch.randperm(d, generator=g)][:, None]
        S[:, :, 3] = 0.0
    return S


# ------------------------------------------------------------------ codec

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("kind", ["normal", "planted", "scaled", "zero"])
@pytest.mark.parametrize("comps", [(2, 2), (0, 0), (4, 4), (1, 3)])
@pytest.mark.parametrize("smooth,select", [(1, "l2"), (0, "l2"), (1, "maxabs")])
def test_prefill_codec_bit_exact(d, kind, comps, smooth, select):
    B, H = 3, 5
    nr, nc = comps
    S0 = _state(kind, 7 + d, B, H, d)
    st = lq.DecodeState(B, H, d, window=16, n_comp_rows=nr, n_comp_cols=nc, smooth=smooth, select=select,
                        device=DEV)
    st.prefill(S0.to(DEV).contiguous())
    torch.cuda.synchronize()
    assert st.device_status() == lq.LQ_OK
    got = snapshot(st)
    p = oracle_params(d, nr=nr, nc=nc, smooth=smooth, select=select)
    for u in range(B * H):
        b, h = divmod(u, H)
        e = oracle.encode(p, S0[b, h].double().numpy())
        np.testing.assert_array_equal(got["codes"][b, h].numpy(), e.Q)
        np.testing.assert_array_equal(got["row_scale"][b, h].numpy(), e.sigma)
        np.testing.assert_array_equal(got["col_smooth"][b, h].numpy(), e.s)
        if nr + nc == 0:
            assert got["comp_index"] is None
            continue
        idx = got["comp_index"][b, h].numpy()
        np.testing.assert_array_equal(idx[:nr], e.comp_rows)
        np.testing.assert_array_equal(idx[nr:nr + nc], e.comp_cols)
        if nr:
            np.testing.assert_array_equal(got["comp_row_vec"][b, h].numpy(), e.row_vecs)
        if nc:
            np.testing.assert_array_equal(got["comp_col_vec"][b, h].numpy(), e.col_vecs)


@pytest.mark.parametrize("d", [64, 128])
def test_naive_prefill_bit_exact(d):
    B, H = 2, 3
    S0 = _state("scaled", 3, B, H, d)
    st = lq.DecodeState(B, H, d, mode="naive", device=DEV)
    st.prefill(S0.to(DEV).contiguous())
    p = oracle_params(d, nr=0, nc=0, smooth=0, mode="naive")
    got = st.export(["codes", "row_scale"])
    for u in range(B * H):
        b, h = divmod(u, H)
        e = oracle.encode(p, S0[b, h].double().numpy())
        np.testing.assert_array_equal(got["codes"][b, h].numpy(), e.Q)
        np.testing.assert_array_equal(got["row_scale"][b, h].numpy(), e.sigma)


# ------------------------------------------------------------ windowed decode

def _window_case(d, gate, dtype, W, nr, nc, B, H, T, seed, S0_kind="zero", smooth=1, select="l2"):
    """Free-running: GPU and oracle each run their own trajectory from the same S0.
    Teacher-forced: every GPU window starts from the oracle's encoded state."""
    tb = inputs.tokens(seed, 0, T, B, H, d, d, per_channel_gate=(gate == "channel"), dtype=dtype)
    tbd = to_device(tb, DEV)
    S0 = _state(S0_kind, seed, B, H, d)
    st = lq.DecodeState(B, H, d, window=W, n_comp_rows=nr, n_comp_cols=nc, gate=gate, in_dtype=dtype,
                        smooth=smooth, select=select, device=DEV)
    st.prefill(S0.to(DEV).contiguous())
    o_free, shots = gpu_run(st, tbd, flush_every=W)
    assert st.device_status() == lq.LQ_OK
    p = oracle_params(d, W, nr, nc, gate, "window", smooth, select)
    q, k, v, g, beta = unit_inputs(tb, range(B * H))
    ref = oracle.run(p, S0.reshape(B * H, d, d).double().numpy(), q, k, v, g, beta)

    # free-running: outputs over the whole run, codes at the first flush
    o_ref = ref.o.reshape(B, H, T, d).transpose(2, 0, 1, 3)
    err = rel_l2(o_free.numpy(), o_ref)
    assert err <= 1e-3, err
    if shots:
        frac, worst = compare_codes(shots[0]["codes"].reshape(B * H, d, d).numpy(), ref.Q[:, 1])
        assert frac >= 0.999 and worst <= 1, ("free-running first flush", frac, worst)

    # teacher-forced: window by window from the oracle's state
    plain = oracle_params(d, gate=gate, mode="fp32")
    st.prefill(None)
    for w in range(T // W):
        import_encoded(st, ref, w)
        sl = slice(w * W, (w + 1) * W)
        o_w, snaps = gpu_run(st, inputs.TokenBatch(*(x[sl] for x in (tbd.q, tbd.k, tbd.v, tbd.g, tbd.beta))),
                             flush_every=W)
        assert st.device_status() == lq.LQ_OK
        e_w = rel_l2(o_w.numpy(), o_ref[sl])
        assert e_w <= 1e-5, ("teacher-forced outputs", w, e_w)
        snap = snaps[0]
        got_idx = snap["comp_index"].reshape(B * H, -1).numpy()[:, :nr + nc] if nr + nc else None
        codes = snap["codes"].reshape(B * H, d, d).numpy()
        keep = np.ones(B * H, bool)
        if nr + nc:
            flips = np.nonzero((got_idx != ref.idx[:, w + 1]).any(axis=1))[0]
            if len(flips):
                S_tilde = decoded_state(ref, w, nr, nc, d)
                pre = oracle.run(plain, S_tilde[flips], q[flips, sl], k[flips, sl], v[flips, sl], g[flips, sl],
                                 beta[flips, sl], snapshots=False).S_final
                for i, n in enumerate(flips):
                    assert selection_is_near_tie(pre[i], got_idx[n], ref.idx[n, w + 1], nr, select), (w, n)
                keep[flips] = False
        frac, worst = compare_codes(codes[keep], ref.Q[keep, w + 1])
        assert frac >= 0.999 and worst <= 1, ("teacher-forced flush", w, frac, worst)
        same_rows = (codes == ref.Q[:, w + 1]).all(axis=2) & keep[:, None]
        sig = snap["row_scale"].reshape(B * H, d).numpy()
        np.testing.assert_allclose(sig[same_rows], ref.sigma[:, w + 1][same_rows], rtol=1e-5)
        if nr + nc:
            np.testing.assert_allclose(snap["col_smooth"].reshape(B * H, d).numpy()[keep],
                                       ref.s[keep, w + 1], rtol=1e-5)
    return err


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_tiny_gdn_workload(dtype):
    """One sequence, one 64x64 head from a zero state, 256 tokens, W = 64, 2+2 compensators."""
    wl = inputs.WORKLOADS["gdn_tiny_d64"]
    _window_case(64, "scalar", dtype, wl.window, wl.n_comp_rows, wl.n_comp_cols, wl.batch, wl.heads,
                 wl.decode_tokens, wl.seed)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("W,nr,nc", [(1, 2, 2), (5, 1, 0), (37, 2, 2), (64, 4, 4)])
def test_window_decode_variants(d, gate, W, nr, nc):
    B, H = 2, 3
    T = 2 * W + W // 2 + 1 if W > 1 else 9
    _window_case(d, gate, torch.bfloat16, W, nr, nc, B, H, T, seed=11 + W, S0_kind="normal")


@pytest.mark.parametrize("W", [128, 256])
def test_window_decode_long_gdn_windows(W):
    """The sweep's longest windows (GDN, d = 128, bf16 inputs, 2 + 2
    compensators): two full windows and half of a third, every window
    teacher-forced from the oracle's encoding."""
    _window_case(128, "scalar", torch.bfloat16, W, 2, 2, 2, 3, 2 * W + W // 2 + 1, seed=13 + W, S0_kind="normal")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_window_decode_fp32_inputs(d, gate):
    """FP32 q, k, v (so FP32 buffered keys): every decode instantiation with FP32 inputs."""
    W = 37
    _window_case(d, gate, torch.float32, W, 2, 2, 2, 3, 2 * W + 5, seed=71, S0_kind="normal")


def test_window_decode_planted_outliers_maxabs_nosmooth():
    d, B, H, W = 128, 2, 4, 16
    for smooth, select in ((0, "l2"), (1, "maxabs")):
        _window_case(d, "scalar", torch.bfloat16, W, 2, 2, B, H, 3 * W, seed=5, S0_kind="planted",
                     smooth=smooth, select=select)


def test_partial_window_flush_and_window_full():
    d, B, H, W = 64, 1, 2, 8
    tb = to_device(inputs.tokens(2, 0, 20, B, H, d, d, per_channel_gate=False), DEV)
    st = lq.DecodeState(B, H, d, window=W, device=DEV)
    st.prefill(None)
    for t in range(W):
        st.decode_step(tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t])
    with pytest.raises(lq.LQError) as ei:
        st.decode_step(tb.q[W], tb.k[W], tb.v[W], tb.g[W], tb.beta[W])
    assert ei.value.status == lq.LQ_ERR_WINDOW_FULL and st.fill == W
    st.flush()
    assert st.fill == 0
    for t in range(W, W + 3):
        st.decode_step(tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t])
    st.flush()          # a partial window
    st.flush()          # an empty one
    assert st.device_status() == lq.LQ_OK


def test_kda_gate_sum_out_of_range_is_reported():
    d, B, H, W = 64, 1, 1, 64
    tb = inputs.tokens(4, 0, W, B, H, d, d, per_channel_gate=True)
    tb.g.fill_(-2.0)                       # G reaches -128 within the window
    tb = to_device(tb, DEV)
    st = lq.DecodeState(B, H, d, window=W, gate="channel", device=DEV)
    st.prefill(None)
    for t in range(W):
        st.decode_step(tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t])
    assert st.device_status() == lq.LQ_ERR_RANGE
    st.prefill(None)                       # prefill clears the error word
    assert st.device_status() == lq.LQ_OK


# ------------------------------------------------------------ comparators

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_fp32_state_decode(d, gate, dtype):
    B, H, T = 2, 3, 96
    tb = inputs.tokens(21, 0, T, B, H, d, d, per_channel_gate=(gate == "channel"), dtype=dtype)
    S0 = _state("normal", 21, B, H, d)
    st = lq.DecodeState(B, H, d, gate=gate, mode="fp32", in_dtype=dtype, device=DEV)
    st.prefill(S0.to(DEV).contiguous())
    o_gpu, _ = gpu_run(st, to_device(tb, DEV))
    ref = oracle.run(oracle_params(d, gate=gate, mode="fp32"), S0.reshape(-1, d, d).double().numpy(),
                     *unit_inputs(tb, range(B * H)))
    o_ref = ref.o.reshape(B, H, T, d).transpose(2, 0, 1, 3)
    assert rel_l2(o_gpu.numpy(), o_ref) <= 1e-5
    S_gpu = st.read("state_f32").reshape(-1, d, d).numpy()
    assert rel_l2(S_gpu, ref.S_final) <= 1e-5


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_naive_int8_decode(d, gate):
    B, H, T = 2, 3, 64
    tb = inputs.tokens(31, 0, T, B, H, d, d, per_channel_gate=(gate == "channel"))
    S0 = _state("normal", 31, B, H, d)
    st = lq.DecodeState(B, H, d, gate=gate, mode="naive", device=DEV)
    st.prefill(S0.to(DEV).contiguous())
    o_gpu, _ = gpu_run(st, to_device(tb, DEV))
    ref = oracle.run(oracle_params(d, gate=gate, mode="naive"), S0.reshape(-1, d, d).double().numpy(),
                     *unit_inputs(tb, range(B * H)))
    o_ref = ref.o.reshape(B, H, T, d).transpose(2, 0, 1, 3)
    assert rel_l2(o_gpu.numpy(), o_ref) <= 1e-3
    # teacher-forced: every token starts from the oracle's requantized state
    tbd = to_device(tb, DEV)
    for t in range(T):
        import_encoded(st, ref, t)
        o_t = st.decode_step(tbd.q[t], tbd.k[t], tbd.v[t], tbd.g[t], tbd.beta[t])
        assert rel_l2(o_t.cpu().numpy(), o_ref[t]) <= 1e-5, t
        frac, worst = compare_codes(st.read("codes").reshape(-1, d, d).numpy(), ref.Q[:, t + 1])
        assert frac >= 0.999 and worst <= 1, (t, frac, worst)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_naive_int8_decode_many_units_per_cta(gate, dtype):
    """The naive kernel is persistent: with 38 x 32 units every CTA walks several
    units through its slot ring.  Sampled units are checked against the oracle,
    free-running and teacher-forced per token."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    d, H, T = 128, 32, 6
    B = -(-8 * sms // H) + 1
    tb = inputs.tokens(33, 0, T, B, H, d, d, per_channel_gate=(gate == "channel"), dtype=dtype)
    S0 = _state("normal", 33, B, H, d)
    st = lq.DecodeState(B, H, d, gate=gate, mode="naive", in_dtype=dtype, device=DEV)
    st.prefill(S0.to(DEV).contiguous())
    o_gpu, _ = gpu_run(st, to_device(tb, DEV))
    assert st.device_status() == lq.LQ_OK
    units = sorted(np.random.default_rng(33).choice(B * H, 8, replace=False).tolist())
    ref = oracle.run(oracle_params(d, gate=gate, mode="naive"), S0.reshape(-1, d, d)[units].double().numpy(),
                     *unit_inputs(tb, units))
    o_s = o_gpu.reshape(T, B * H, d)[:, units].transpose(0, 1).numpy()
    assert rel_l2(o_s, ref.o) <= 1e-3
    tbd = to_device(tb, DEV)
    st.prefill(S0.to(DEV).contiguous())
    for t in range(T):
        import_encoded(st, ref, t, units)
        o_t = st.decode_step(tbd.q[t], tbd.k[t], tbd.v[t], tbd.g[t], tbd.beta[t])
        got = o_t.reshape(B * H, d)[units].cpu().numpy()
        assert rel_l2(got, ref.o[:, t]) <= 1e-5, t
        codes = st.read("codes").reshape(B * H, d, d)[units].numpy()
        frac, worst = compare_codes(codes, ref.Q[:, t + 1])
        assert frac >= 0.999 and worst <= 1, (t, frac, worst)
