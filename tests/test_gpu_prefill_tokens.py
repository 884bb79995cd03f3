"""Prefill from prompt tokens on the GPU against the oracle.

The recurrence part is checked against the oracle's dense FP64 recurrence
(its FP32-state mode: the gated delta rule of Gated DeltaNet / Kimi Delta
Attention with no quantization), the codec part bit for bit against the
oracle's encoder applied to the kernel's own FP32 final state, which an FP32
handle of the same kernel exposes (the codec of LeapQuant, "LeapQuant:
Efficient Linear Attention with Accurate Recurrent State Quantization",
section "Abstract (arXiv)").
"""
import numpy as np
import pytest
import torch

import oracle
from harness import oracle_params, rel_l2, selection_is_near_tie, snapshot, to_device, unit_inputs
from recurrent_state_quantization_lq_b200 import inputs, lq

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _prompt(d, gate, dtype, B, H, T, seed, with_s0=True):
    tb = inputs.tokens(seed, 0, T, B, H, d, d, gate == "channel", dtype)
    S0 = 0.5 * torch.randn(B, H, d, d, generator=torch.Generator().manual_seed(seed)) if with_s0 else None
    return tb, S0


def _gpu_prefill(mode, d, gate, dtype, tb, S0, nr=2, nc=2, outputs=True):
    T, B, H = tb.q.shape[:3]
    st = lq.DecodeState(B, H, d, window=16, n_comp_rows=nr, n_comp_cols=nc, gate=gate, mode=mode, in_dtype=dtype,
                        device=DEV)
    tbd = to_device(tb, DEV)
    out = torch.full((T, B, H, d), float("nan"), device=DEV) if outputs else None
    st.prefill_tokens(tbd.q, tbd.k, tbd.v, tbd.g, tbd.beta, S0=None if S0 is None else S0.to(DEV).contiguous(),
                      out=out)
    assert st.device_status() == lq.LQ_OK, lq.last_error()
    return st, out


@pytest.mark.parametrize("d,gate,dtype", [(64, "scalar", torch.bfloat16), (128, "scalar", torch.bfloat16),
                                          (128, "channel", torch.bfloat16), (64, "channel", torch.float32),
                                          (128, "scalar", torch.float32)])
@pytest.mark.parametrize("T", [1, 17, 40])
def test_recurrence_matches_fp64(d, gate, dtype, T):
    B, H = 2, 3
    tb, S0 = _prompt(d, gate, dtype, B, H, T, seed=100 + T)
    st, out = _gpu_prefill("fp32", d, gate, dtype, tb, S0)
    p = oracle_params(d, gate=gate, mode="fp32")
    q, k, v, g, beta = unit_inputs(tb, range(B * H))
    r = oracle.run(p, S0.double().numpy().reshape(B * H, d, d), q, k, v, g, beta, snapshots=False)
    S_gpu = st.read("state_f32").double().numpy().reshape(B * H, d, d)
    o_gpu = out.cpu().double().numpy().reshape(T, B * H, d).transpose(1, 0, 2)
    # FP32 arithmetic against FP64: a few ulps per step, well under the 1e-3 target
    assert rel_l2(S_gpu, r.S_final) <= 1e-5
    assert rel_l2(o_gpu, r.o) <= 1e-5
    for u in range(B * H):
        assert rel_l2(o_gpu[u], r.o[u]) <= 1e-5, u


@pytest.mark.parametrize("d,gate", [(64, "scalar"), (128, "scalar"), (128, "channel")])
@pytest.mark.parametrize("comps", [(2, 2), (0, 0), (3, 1)])
def test_codec_on_the_final_state_bit_exact(d, gate, comps):
    B, H, T = 3, 2, 23
    nr, nc = comps
    tb, S0 = _prompt(d, gate, torch.bfloat16, B, H, T, seed=7 + d)
    ref, _ = _gpu_prefill("fp32", d, gate, torch.bfloat16, tb, S0, outputs=False)
    st, _ = _gpu_prefill("window", d, gate, torch.bfloat16, tb, S0, nr=nr, nc=nc, outputs=False)
    S = ref.read("state_f32")
    got = snapshot(st)
    p = oracle_params(d, nr=nr, nc=nc, gate=gate)
    for u in range(B * H):
        b, h = divmod(u, H)
        e = oracle.encode(p, S[b, h].double().numpy())
        if nr + nc:
            idx = got["comp_index"][b, h].numpy()
            if not (np.array_equal(idx[:nr], e.comp_rows) and np.array_equal(idx[nr:nr + nc], e.comp_cols)):
                ref_idx = np.concatenate([e.comp_rows, e.comp_cols])
                assert selection_is_near_tie(S[b, h].double().numpy(), idx[:nr + nc], ref_idx, nr), u
                continue
        np.testing.assert_array_equal(got["codes"][b, h].numpy(), e.Q)
        np.testing.assert_array_equal(got["row_scale"][b, h].numpy(), e.sigma)
        np.testing.assert_array_equal(got["col_smooth"][b, h].numpy(), e.s)


@pytest.mark.parametrize("gate", ["scalar", "channel"])
def test_decode_after_prompt_equals_ingested_state(gate):
    """Prefill from tokens, then decode, equals ingesting the same FP32 state
    with lq_prefill_state and decoding: outputs identical bit for bit."""
    d, B, H, T, W = 128, 2, 3, 37, 8
    tb, S0 = _prompt(d, gate, torch.bfloat16, B, H, T, seed=61)
    ref, _ = _gpu_prefill("fp32", d, gate, torch.bfloat16, tb, S0, outputs=False)
    a = lq.DecodeState(B, H, d, window=W, gate=gate, device=DEV)
    b = lq.DecodeState(B, H, d, window=W, gate=gate, device=DEV)
    tbd = to_device(tb, DEV)
    a.prefill_tokens(tbd.q, tbd.k, tbd.v, tbd.g, tbd.beta, S0=S0.to(DEV).contiguous())
    b.prefill(ref.read("state_f32", device=DEV))
    dec = to_device(inputs.tokens(62, 0, 2 * W, B, H, d, d, gate == "channel"), DEV)
    for t in range(2 * W):
        oa = a.decode_step(dec.q[t], dec.k[t], dec.v[t], dec.g[t], dec.beta[t])
        ob = b.decode_step(dec.q[t], dec.k[t], dec.v[t], dec.g[t], dec.beta[t])
        assert torch.equal(oa, ob), t
        if a.fill == W:
            a.flush()
            b.flush()
    assert a.device_status() == lq.LQ_OK and b.device_status() == lq.LQ_OK


def test_zero_tokens_and_zero_state():
    d, B, H = 64, 2, 2
    tb, S0 = _prompt(d, "scalar", torch.bfloat16, B, H, 4, seed=3)
    a = lq.DecodeState(B, H, d, window=8, device=DEV)
    b = lq.DecodeState(B, H, d, window=8, device=DEV)
    tbd = to_device(tb, DEV)
    a.prefill_tokens(tbd.q[:0], tbd.k[:0], tbd.v[:0], tbd.g[:0], tbd.beta[:0], S0=S0.to(DEV).contiguous())
    b.prefill(S0.to(DEV).contiguous())
    for name in ("codes", "row_scale", "col_smooth", "comp_index", "comp_row_vec", "comp_col_vec"):
        assert torch.equal(a.read(name), b.read(name)), name
    # from a zero state, a prompt of one token: S_1 = beta_1 v_1 k_1^T, o_1 = S_1 q_1
    z = lq.DecodeState(B, H, d, mode="fp32", device=DEV)
    out = torch.empty(1, B, H, d, device=DEV)
    z.prefill_tokens(tbd.q[:1], tbd.k[:1], tbd.v[:1], tbd.g[:1], tbd.beta[:1], out=out)
    k1, v1, q1 = (x[0].float().cpu() for x in (tb.k, tb.v, tb.q))
    S1 = tb.beta[0][..., None, None] * v1[..., :, None] * k1[..., None, :]
    assert torch.allclose(z.read("state_f32"), S1, rtol=1e-6, atol=1e-7)
    assert torch.allclose(out[0].cpu(), (S1 @ q1[..., None])[..., 0], rtol=1e-5, atol=1e-6)


def test_ragged_handle_counts_cleared():
    d, B, H, W = 64, 3, 2, 4
    st = lq.DecodeState(B, H, d, window=W, ragged=True, device=DEV)
    st.prefill(None)
    dec = to_device(inputs.tokens(9, 0, 3, B, H, d, d, False), DEV)
    for t in range(3):
        st.decode_step(dec.q[t], dec.k[t], dec.v[t], dec.g[t], dec.beta[t],
                       active=torch.tensor([1, 0, 1], dtype=torch.uint8, device=DEV))
    tb = to_device(inputs.tokens(10, 0, 5, B, H, d, d, False), DEV)
    st.prefill_tokens(tb.q, tb.k, tb.v, tb.g, tb.beta)
    assert st.device_status() == lq.LQ_OK
    assert int(st.fills().abs().sum()) == 0


def test_full_size_prompt_sampled_units():
    """The 64 x 32 x 128 GDN workload's 512-token prompt, as bench.py runs it:
    outputs and final states of sampled units against the oracle."""
    B, H, d, T = 64, 32, 128, 512
    tb = inputs.tokens(5, 0, T, B, H, d, d, False, torch.bfloat16)
    st = lq.DecodeState(B, H, d, mode="fp32", device=DEV)
    tbd = to_device(tb, DEV)
    out = torch.empty(T, B, H, d, device=DEV)
    st.prefill_tokens(tbd.q, tbd.k, tbd.v, tbd.g, tbd.beta, out=out)
    assert st.device_status() == lq.LQ_OK
    assert bool(torch.isfinite(out).all())
    rng = np.random.default_rng(0)
    units = sorted(set(rng.integers(0, B * H, 12).tolist()) | {0, B * H - 1})
    p = oracle_params(d, mode="fp32")
    q, k, v, g, beta = unit_inputs(tb, units)
    r = oracle.run(p, np.zeros((len(units), d, d)), q, k, v, g, beta, snapshots=False)
    S_gpu = st.read("state_f32").reshape(B * H, d, d)[units].double().numpy()
    o_gpu = out.reshape(T, B * H, d)[:, units].cpu().double().numpy().transpose(1, 0, 2)
    assert rel_l2(S_gpu, r.S_final) <= 1e-5
    assert rel_l2(o_gpu, r.o) <= 1e-5


@pytest.mark.parametrize("d", [64, 128])
def test_naive_mode_codec_on_the_final_state(d):
    """Naive per-token INT8 handles encode the prompt's final state with their
    own codec (no compensators, no smoothing), bit for bit."""
    B, H, T = 2, 3, 19
    tb, S0 = _prompt(d, "scalar", torch.bfloat16, B, H, T, seed=29 + d)
    ref, _ = _gpu_prefill("fp32", d, "scalar", torch.bfloat16, tb, S0, outputs=False)
    st, _ = _gpu_prefill("naive", d, "scalar", torch.bfloat16, tb, S0, outputs=False)
    S = ref.read("state_f32")
    p = oracle_params(d, nr=0, nc=0, smooth=0, mode="naive")
    got = st.export(["codes", "row_scale"])
    got_c, got_s = got["codes"], got["row_scale"]
    for u in range(B * H):
        b, h = divmod(u, H)
        e = oracle.encode(p, S[b, h].double().numpy())
        np.testing.assert_array_equal(got_c[b, h].numpy(), e.Q)
        np.testing.assert_array_equal(got_s[b, h].numpy(), e.sigma)
