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

from harness import compare_codes, gpu_run, oracle_params, rel_l2, snapshot, to_device, unit_inputs

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
    for u in range(B * H):
        b, h = divmod(u, H)
        e = oracle.encode(p, S0[b, h].double().numpy())
        np.testing.assert_array_equal(st.view("codes")[b, h].cpu().numpy(), e.Q)
        np.testing.assert_array_equal(st.view("row_scale")[b, h].cpu().numpy(), e.sigma)


# ------------------------------------------------------------ windowed decode

def _window_case(d, gate, dtype, W, nr, nc, B, H, T, seed, S0_kind="zero", smooth=1, select="l2"):
    tb = inputs.tokens(seed, 0, T, B, H, d, d, per_channel_gate=(gate == "channel"), dtype=dtype)
    S0 = _state(S0_kind, seed, B, H, d)
    st = lq.DecodeState(B, H, d, window=W, n_comp_rows=nr, n_comp_cols=nc, gate=gate, in_dtype=dtype,
                        smooth=smooth, select=select, device=DEV)
    st.prefill(S0.to(DEV).contiguous())
    o_gpu, shots = gpu_run(st, to_device(tb, DEV), flush_every=W)
    assert st.device_status() == lq.LQ_OK
    p = oracle_params(d, W, nr, nc, gate, "window", smooth, select)
    units = range(B * H)
    q, k, v, g, beta = unit_inputs(tb, units)
    ref = oracle.run(p, S0.reshape(B * H, d, d).double().numpy(), q, k, v, g, beta)
    return o_gpu, shots, ref


def _check_window(o_gpu, shots, ref, B, H, d, out_tol=1e-3):
    T = o_gpu.shape[0]
    o_ref = ref.o.reshape(B, H, T, d).transpose(2, 0, 1, 3)
    err = rel_l2(o_gpu.numpy(), o_ref)
    assert err <= out_tol, err
    for f, snap in enumerate(shots):
        q_gpu = snap["codes"].reshape(B * H, d, d).numpy()
        q_ref = ref.Q[:, f + 1]
        frac, worst = compare_codes(q_gpu, q_ref)
        assert frac >= 0.999 and worst <= 1, (f, frac, worst)
        same = q_gpu == q_ref
        sig_g = snap["row_scale"].reshape(B * H, d).numpy()
        rows_same = same.all(axis=2)
        np.testing.assert_allclose(sig_g[rows_same], ref.sigma[:, f + 1][rows_same], rtol=1e-4)
    return err


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_tiny_gdn_workload(dtype):
    """One sequence, one 64x64 head from a zero state, 256 tokens, W = 64, 2+2 compensators."""
    wl = inputs.WORKLOADS["gdn_tiny_d64"]
    o_gpu, shots, ref = _window_case(64, "scalar", dtype, wl.window, wl.n_comp_rows, wl.n_comp_cols,
                                     wl.batch, wl.heads, wl.decode_tokens, wl.seed)
    assert len(shots) == 4
    _check_window(o_gpu, shots, ref, 1, 1, 64)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("W,nr,nc", [(1, 2, 2), (5, 1, 0), (37, 2, 2), (64, 4, 4)])
def test_window_decode_variants(d, gate, W, nr, nc):
    B, H = 2, 3
    T = 2 * W + W // 2 + 1 if W > 1 else 9
    o_gpu, shots, ref = _window_case(d, gate, torch.bfloat16, W, nr, nc, B, H, T, seed=11 + W,
                                     S0_kind="normal")
    _check_window(o_gpu, shots, ref, B, H, d)


def test_window_decode_planted_outliers_maxabs_nosmooth():
    d, B, H, W = 128, 2, 4, 16
    for smooth, select in ((0, "l2"), (1, "maxabs")):
        o_gpu, shots, ref = _window_case(d, "scalar", torch.bfloat16, W, 2, 2, B, H, 3 * W, seed=5,
                                         S0_kind="planted", smooth=smooth, select=select)
        _check_window(o_gpu, shots, ref, B, H, d)


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
    S_gpu = st.view("state_f32").reshape(-1, d, d).cpu().numpy()
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
    frac, worst = compare_codes(st.view("codes").reshape(-1, d, d).cpu().numpy(), ref.Q[:, -1])
    assert frac >= 0.999 and worst <= 1, (frac, worst)
