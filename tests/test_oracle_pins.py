"""Pins of the CPU oracle against facts fixed by the mathematics (CPU only).

Each test checks the oracle against something other than itself: identities
of the delta rule, closed forms, hand-worked examples under tests/golden/,
the codec's round-trip bound and the error bound of the windowed scheme.
"""
import os

import numpy as np
import pytest

import oracle
from oracle import GATE_CHANNEL, GATE_SCALAR, MODE_FP32, MODE_NAIVE, MODE_WINDOW, Params

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _unit(rng, d):
    x = rng.standard_normal(d)
    return x / np.linalg.norm(x)


def _read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows[key] = vals
    return rows


# ---------------------------------------------------------------- recurrence

@pytest.mark.parametrize("gate", [GATE_SCALAR, GATE_CHANNEL])
def test_worked_example(gate):
    """Hand-derived single token (tests/golden/recurrence_worked_example.txt)."""
    rows = _read_golden("recurrence_worked_example.txt")
    key = "gdn" if gate == GATE_SCALAR else "kda"
    alpha_s, *rest = rows[key]
    alpha = np.array([float(a) for a in alpha_s.split(",")])
    vals = np.array([float(x) for x in rest])
    S_exp, o_exp = vals[:4].reshape(2, 2), vals[4:]
    p = Params(d_k=2, d_v=2, gate=gate, mode=MODE_FP32)
    S = np.array([[1.0, 2.0], [3.0, 4.0]])
    S1, o = oracle.step(p, S, q=[1, 1], k=[0.6, 0.8], v=[1, -1], g=np.log(alpha), beta=0.5)
    np.testing.assert_allclose(S1, S_exp, atol=1e-14)
    np.testing.assert_allclose(o, o_exp, atol=1e-14)


@pytest.mark.parametrize("gate", [GATE_SCALAR, GATE_CHANNEL])
@pytest.mark.parametrize("d", [(8, 5), (64, 64)])
def test_delta_rule_writes_v_at_k(gate, d):
    """beta = 1, |k| = 1: the delta rule stores v exactly at key k, S_t k = v,
    whatever the previous state and the gate."""
    dk, dv = d
    rng = np.random.default_rng(1)
    p = Params(d_k=dk, d_v=dv, gate=gate, mode=MODE_FP32)
    S = rng.standard_normal((dv, dk))
    k = _unit(rng, dk)
    v = rng.standard_normal(dv)
    g = -rng.uniform(0.01, 0.5, 1 if gate == GATE_SCALAR else dk)
    S1, o = oracle.step(p, S, q=k, k=k, v=v, g=g, beta=1.0)
    np.testing.assert_allclose(S1 @ k, v, atol=1e-12)
    np.testing.assert_allclose(o, v, atol=1e-12)   # o = S_t q with q = k


@pytest.mark.parametrize("gate", [GATE_SCALAR, GATE_CHANNEL])
def test_general_beta_along_k(gate):
    """|k| = 1: along k the new state mixes the gated old read-out and v with
    weights (1 - beta) and beta."""
    dk, dv = 12, 7
    rng = np.random.default_rng(2)
    p = Params(d_k=dk, d_v=dv, gate=gate, mode=MODE_FP32)
    S = rng.standard_normal((dv, dk))
    k = _unit(rng, dk)
    v = rng.standard_normal(dv)
    beta = 0.3
    g = -rng.uniform(0.01, 0.5, 1 if gate == GATE_SCALAR else dk)
    alpha = np.exp(g) * np.ones(dk)
    S1, _ = oracle.step(p, S, q=k, k=k, v=v, g=g, beta=beta)
    np.testing.assert_allclose(S1 @ k, (1 - beta) * (S @ (alpha * k)) + beta * v, atol=1e-12)


@pytest.mark.parametrize("gate", [GATE_SCALAR, GATE_CHANNEL])
def test_orthogonal_complement_only_decays(gate):
    """For x orthogonal to k the update only applies the gate: S_t x = S diag(alpha) x.
    Together with the test above this fixes S_t on all of R^{d_k}."""
    dk, dv = 10, 6
    rng = np.random.default_rng(3)
    p = Params(d_k=dk, d_v=dv, gate=gate, mode=MODE_FP32)
    S = rng.standard_normal((dv, dk))
    k = _unit(rng, dk)
    x = rng.standard_normal(dk)
    x -= (x @ k) * k
    g = -rng.uniform(0.01, 0.5, 1 if gate == GATE_SCALAR else dk)
    alpha = np.exp(g) * np.ones(dk)
    S1, o = oracle.step(p, S, q=x, k=k, v=rng.standard_normal(dv), g=g, beta=0.7)
    # S_t x = S diag(alpha)(I - beta k k^T) x + beta v (k.x) = S diag(alpha) x when k.x = 0
    np.testing.assert_allclose(S1 @ x, S @ (alpha * x), atol=1e-12)
    np.testing.assert_allclose(o, S1 @ x, atol=1e-12)


def test_kda_equal_gates_is_gdn():
    dk, dv, T = 16, 9, 20
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, T, dk))
    k = np.stack([_unit(rng, dk) for _ in range(T)])[None]
    v = rng.standard_normal((1, T, dv))
    g = -rng.uniform(0.01, 0.3, (1, T))
    beta = rng.uniform(0.1, 0.9, (1, T))
    S0 = rng.standard_normal((1, dv, dk))
    a = oracle.run(Params(dk, dv, gate=GATE_SCALAR, mode=MODE_FP32), S0, q, k, v, g, beta)
    b = oracle.run(Params(dk, dv, gate=GATE_CHANNEL, mode=MODE_FP32), S0, q, k, v,
                   np.repeat(g[..., None], dk, axis=-1), beta)
    np.testing.assert_allclose(a.o, b.o, atol=1e-12)
    np.testing.assert_allclose(a.S_final, b.S_final, atol=1e-12)


@pytest.mark.parametrize("gate", [GATE_SCALAR, GATE_CHANNEL])
def test_beta_zero_closed_form(gate):
    """beta = 0: S_T = S_0 diag(exp(sum_t g_t)) and o_t = S_t q_t."""
    dk, dv, T = 8, 6, 30
    rng = np.random.default_rng(5)
    gd = 1 if gate == GATE_SCALAR else dk
    q = rng.standard_normal((1, T, dk))
    k = rng.standard_normal((1, T, dk))
    v = rng.standard_normal((1, T, dv))
    g = -rng.uniform(0.0, 0.2, (1, T, gd))
    S0 = rng.standard_normal((1, dv, dk))
    r = oracle.run(Params(dk, dv, gate=gate, mode=MODE_FP32), S0, q, k, v, g, np.zeros((1, T)))
    G = np.cumsum(g[0], axis=0) * np.ones((T, dk))
    for t in range(T):
        np.testing.assert_allclose(r.o[0, t], (S0[0] * np.exp(G[t])[None, :]) @ q[0, t], atol=1e-12)
    np.testing.assert_allclose(r.S_final[0], S0[0] * np.exp(G[-1])[None, :], atol=1e-12)


def test_orthonormal_keys_build_columns():
    """alpha = 1, beta = 1, S_0 = 0, k_t = e_t: the state's column t is v_t."""
    d, dv = 6, 4
    rng = np.random.default_rng(6)
    k = np.eye(d)[None]
    v = rng.standard_normal((1, d, dv))
    q = rng.standard_normal((1, d, d))
    r = oracle.run(Params(d, dv, mode=MODE_FP32), np.zeros((1, dv, d)), q, k, v,
                   np.zeros((1, d)), np.ones((1, d)))
    np.testing.assert_allclose(r.S_final[0], v[0].T, atol=1e-14)
    for t in range(d):
        np.testing.assert_allclose(r.o[0, t], v[0, :t + 1].T @ q[0, t, :t + 1], atol=1e-13)


# --------------------------------------------------------------------- codec

def test_codec_worked_example():
    rows = _read_golden("codec_worked_example.txt")
    f = lambda key: np.array([float(x) for x in rows[key]])
    S = f("state").reshape(3, 4)
    p = Params(d_k=4, d_v=3, n_comp_rows=1, n_comp_cols=1)
    for select in (oracle.SELECT_L2, oracle.SELECT_MAXABS):
        e = oracle.encode(p, S, select=select)
        assert list(e.comp_rows) == [int(x) for x in rows["comp_rows"]]
        assert list(e.comp_cols) == [int(x) for x in rows["comp_cols"]]
        np.testing.assert_array_equal(e.row_vecs.ravel(), f("row_vecs"))
        np.testing.assert_array_equal(e.col_vecs.ravel(), f("col_vecs"))
        np.testing.assert_array_equal(e.s, f("s").astype(np.float32))
        sig = (f("sigma_num").astype(np.float32) / np.float32(127.0)).astype(np.float32)
        np.testing.assert_array_equal(e.sigma, sig)
        np.testing.assert_array_equal(e.Q.ravel(), f("codes").astype(np.int8))
    e = oracle.encode(p, S, smooth=0)
    np.testing.assert_array_equal(e.s, np.ones(4, np.float32))
    sig = (f("sigma_num_nosmooth").astype(np.float32) / np.float32(127.0)).astype(np.float32)
    np.testing.assert_array_equal(e.sigma, sig)
    np.testing.assert_array_equal(e.Q.ravel(), f("codes_nosmooth").astype(np.int8))


@pytest.mark.parametrize("smooth", [0, 1])
def test_codec_rank1_closed_form(smooth):
    """S = a b^T, no compensators.  With smoothing every code is
    sgn(a_i) rint(127 sgn(b_j) sqrt(|b_j| / max|b|)); without it,
    sgn(a_i) rint(127 b_j / max|b|).  b is chosen so the codes are integers n_j."""
    rng = np.random.default_rng(7)
    dv, dk = 9, 16
    n = rng.integers(-127, 128, dk)
    n[0] = 127
    B = 3.7
    b = B * np.sign(n) * (np.abs(n) / 127.0) ** (2 if smooth else 1)
    a = rng.uniform(0.5, 3.0, dv) * rng.choice([-1, 1], dv)
    p = Params(d_k=dk, d_v=dv, n_comp_rows=0, n_comp_cols=0, smooth=smooth)
    e = oracle.encode(p, np.outer(a, b))
    np.testing.assert_array_equal(e.Q, (np.sign(a)[:, None] * n[None, :]).astype(np.int8))


def _roundtrip_check(p, S):
    e = oracle.encode(p, S)
    R32 = S.astype(np.float32).astype(np.float64)
    err = np.abs(R32 - e.S_tilde)
    bound = 0.5 * e.sigma.astype(np.float64)[:, None] * e.s.astype(np.float64)[None, :] * (1 + 1e-6)
    bound += 1e-6 * np.abs(R32)       # FP32 rounding of the scaled residual
    assert np.all(err <= bound + 1e-30)
    assert np.all(np.abs(e.Q.astype(int)) <= 127)
    for i in e.comp_rows:
        np.testing.assert_array_equal(e.S_tilde[i], R32[i])
    for j in e.comp_cols:
        np.testing.assert_array_equal(e.S_tilde[:, j], R32[:, j])
    live = (e.sigma > 0)
    assert np.all(np.abs(e.Q[live]).max(axis=1) == 127)
    return e


@pytest.mark.parametrize("smooth", [0, 1])
@pytest.mark.parametrize("select", [oracle.SELECT_L2, oracle.SELECT_MAXABS])
def test_codec_roundtrip_bound(smooth, select):
    """|S - (sigma_i Q_ij s_j + C_ij)| <= sigma_i s_j / 2 everywhere, exact on the
    compensator rows and columns, codes in [-127, 127], 127 reached in every live row."""
    rng = np.random.default_rng(8)
    for dv, dk, nr, nc in [(64, 64, 2, 2), (128, 128, 4, 4), (17, 33, 1, 3)]:
        p = Params(d_k=dk, d_v=dv, n_comp_rows=nr, n_comp_cols=nc, smooth=smooth, select=select)
        S = rng.standard_normal((dv, dk)) * rng.uniform(0.1, 10, dv)[:, None]
        _roundtrip_check(p, S)


def test_codec_zero_state():
    p = Params(d_k=16, d_v=16)
    e = oracle.encode(p, np.zeros((16, 16)))
    assert not e.Q.any() and not e.sigma.any() and not e.S_tilde.any()
    np.testing.assert_array_equal(e.s, np.ones(16, np.float32))
    assert list(e.comp_rows) == [0, 1] and list(e.comp_cols) == [0, 1]


def test_codec_power_of_two_scale_invariance():
    """Scaling the state by 4 scales sigma by 2 and s by 2 and leaves the codes."""
    rng = np.random.default_rng(9)
    p = Params(d_k=32, d_v=32)
    S = rng.standard_normal((32, 32))
    e1, e4 = oracle.encode(p, S), oracle.encode(p, 4 * S)
    np.testing.assert_array_equal(e1.Q, e4.Q)
    live = np.ones(32, bool)
    live[e1.comp_cols] = False        # extracted columns are empty: s_j = 1 in both
    np.testing.assert_array_equal(2 * e1.s[live], e4.s[live])
    np.testing.assert_array_equal(e1.s[~live], e4.s[~live])
    np.testing.assert_array_equal(2 * e1.sigma, e4.sigma)


def _definition_quantizer(S, comp_rows, comp_cols, smooth):
    """The codec's quantizer written as its definition, in FP64, from the FP32
    residual R (the state with the compensator rows and columns zeroed):
    s_j = sqrt(max_i |R_ij|) (1 for an empty column, or without smoothing),
    R' = R / s, sigma_i = max_j |R'_ij| / 127, Q = clamp(rint(R' / sigma), +-127)
    with Q_i = 0 where sigma_i = 0.  Nothing here calls the oracle."""
    R = S.astype(np.float32).astype(np.float64)
    R[list(comp_rows), :] = 0.0
    R[:, list(comp_cols)] = 0.0
    m = np.abs(R).max(axis=0)
    s = np.where((m > 0) & bool(smooth), np.sqrt(m), 1.0)
    Rp = R / s[None, :]
    sigma = np.abs(Rp).max(axis=1) / 127.0
    with np.errstate(divide="ignore", invalid="ignore"):
        Q = np.where(sigma[:, None] > 0, np.rint(Rp / sigma[:, None]), 0.0)
    return np.clip(Q, -127, 127).astype(np.int32), sigma, s


@pytest.mark.parametrize("smooth", [0, 1])
@pytest.mark.parametrize("kind", ["normal", "scaled", "planted"])
def test_quantizer_reading_within_the_definition_bar(kind, smooth):
    """The oracle applies 1/s_j and 127/M_i as FP32 reciprocal products; the
    definition divides.  Both must give the same codes within the parity bar of
    the method (>= 99.9 % equal, never more than 1 LSB apart) and the same
    scales to FP32 rounding, on normal states, rows spanning six decades
    (with an empty column) and planted outliers."""
    from recurrent_state_quantization_lq_b200 import inputs
    rng = np.random.default_rng(21 + smooth)
    d = 128
    cases = []
    for n in range(6):
        if kind == "normal":
            S = rng.standard_normal((d, d))
        elif kind == "scaled":
            S = rng.standard_normal((d, d)) * np.logspace(-3, 3, d)[rng.permutation(d)][:, None]
            S[:, 3] = 0.0
        else:
            S = inputs.planted_state(40 + n, 1, 1, d, d)[0][0, 0].double().numpy()
        cases.append(S)
    equal, total, worst = 0, 0, 0
    for S in cases:
        for nr, nc in ((2, 2), (0, 0), (4, 4)):
            p = Params(d_k=d, d_v=d, n_comp_rows=nr, n_comp_cols=nc, smooth=smooth)
            e = oracle.encode(p, S)
            Qd, sig_d, s_d = _definition_quantizer(S, e.comp_rows, e.comp_cols, smooth)
            diff = np.abs(e.Q.astype(np.int32) - Qd)
            equal += int((diff == 0).sum())
            total += diff.size
            worst = max(worst, int(diff.max()))
            # s_j is a correctly rounded square root of an FP32 value: exact
            np.testing.assert_array_equal(e.s, s_d.astype(np.float32))
            np.testing.assert_allclose(e.sigma, sig_d, rtol=1e-6, atol=0)
    assert worst <= 1, worst
    assert equal / total >= 0.999, equal / total


def test_planted_outliers_selected():
    """N(0,1) state with 2 rows and 2 columns x50: L2 ranking finds all four."""
    from recurrent_state_quantization_lq_b200 import inputs
    S, rows, cols = inputs.planted_state(seed=3, batch=4, heads=3, d_v=128, d_k=128)
    p = Params(d_k=128, d_v=128)
    for b in range(4):
        for h in range(3):
            e = _roundtrip_check(p, S[b, h].double().numpy())
            assert sorted(e.comp_rows) == sorted(rows[b, h].tolist())
            assert sorted(e.comp_cols) == sorted(cols[b, h].tolist())


# ------------------------------------------------------------ windowed scheme

def _seq(rng, n, T, dk, dv, gate):
    q = np.stack([[_unit(rng, dk) for _ in range(T)] for _ in range(n)])
    k = np.stack([[_unit(rng, dk) for _ in range(T)] for _ in range(n)])
    v = rng.standard_normal((n, T, dv))
    gd = 1 if gate == GATE_SCALAR else dk
    g = -0.1 * np.log1p(np.exp(rng.standard_normal((n, T, gd))))
    beta = 1 / (1 + np.exp(-rng.standard_normal((n, T))))
    return q, k, v, g, beta


@pytest.mark.parametrize("gate", [GATE_SCALAR, GATE_CHANNEL])
def test_single_window_from_zero_is_exact(gate):
    """S_0 = 0 encodes exactly and no flush happens before the last token, so a
    window covering the whole sequence reproduces the unquantized outputs."""
    rng = np.random.default_rng(10)
    n, T, d = 2, 40, 16
    q, k, v, g, beta = _seq(rng, n, T, d, d, gate)
    S0 = np.zeros((n, d, d))
    a = oracle.run(Params(d, d, window=T, gate=gate, mode=MODE_WINDOW), S0, q, k, v, g, beta)
    b = oracle.run(Params(d, d, gate=gate, mode=MODE_FP32), S0, q, k, v, g, beta)
    np.testing.assert_array_equal(a.o, b.o)


@pytest.mark.parametrize("gate", [GATE_SCALAR, GATE_CHANNEL])
@pytest.mark.parametrize("mode", [MODE_WINDOW, MODE_NAIVE])
def test_quantized_error_bound(gate, mode):
    """With alpha <= 1, 0 <= beta <= 1 and |k| = 1 every transition is a
    contraction, so the state error after any token is at most the sum of the
    codec errors made so far, each at most ||sigma s^T / 2||_F."""
    rng = np.random.default_rng(11)
    n, T, d, W = 2, 96, 32, 16
    q, k, v, g, beta = _seq(rng, n, T, d, d, gate)
    S0 = rng.standard_normal((n, d, d))
    p = Params(d, d, window=W, gate=gate, mode=mode)
    rq = oracle.run(p, S0, q, k, v, g, beta)
    rf = oracle.run(Params(d, d, gate=gate, mode=MODE_FP32), S0, q, k, v, g, beta)
    step = 1 if mode == MODE_NAIVE else W
    for h in range(n):
        def codec_bound(f):
            sig = rq.sigma[h, f].astype(np.float64)
            s = rq.s[h, f].astype(np.float64) if mode == MODE_WINDOW else np.ones(d)
            return 0.5 * np.linalg.norm(np.outer(sig, s)) * (1 + 1e-6) + 1e-6 * 10 * d
        total = codec_bound(0)
        for t in range(T):
            diff = np.linalg.norm(rq.o[h, t] - rf.o[h, t])
            assert diff <= total * np.linalg.norm(q[h, t]) + 1e-9
            if (t + 1) % step == 0:
                total += codec_bound((t + 1) // step)
        assert np.linalg.norm(rq.S_final[h] - rf.S_final[h]) <= total + 1e-9


def test_error_ordering_windowed_beats_naive():
    """The windowed codec with compensators and smoothing tracks the unquantized
    outputs more closely than per-token requantization, on the tiny workload's
    recipe and on a planted-outlier state."""
    from recurrent_state_quantization_lq_b200 import inputs
    import torch
    for planted in (False, True):
        n, T, d = 4, 256, 64
        tb = inputs.tokens(0, 0, T, 1, n, d, d, per_channel_gate=False, dtype=torch.float32)
        q, k, v = (x[:, 0].permute(1, 0, 2).double().numpy() for x in (tb.q, tb.k, tb.v))
        g = tb.g[:, 0].permute(1, 0).double().numpy()
        beta = tb.beta[:, 0].permute(1, 0).double().numpy()
        if planted:
            S0 = inputs.planted_state(3, 1, n, d, d)[0][0].double().numpy()
        else:
            S0 = np.zeros((n, d, d))
        ref = oracle.run(Params(d, d, mode=MODE_FP32), S0, q, k, v, g, beta).o
        err = {}
        for mode in (MODE_WINDOW, MODE_NAIVE):
            o = oracle.run(Params(d, d, window=64, mode=mode), S0, q, k, v, g, beta).o
            err[mode] = np.linalg.norm(o - ref) / np.linalg.norm(ref)
        assert err[MODE_WINDOW] < err[MODE_NAIVE], err


def test_naive_is_window_one_without_compensators():
    rng = np.random.default_rng(12)
    n, T, d = 2, 20, 16
    q, k, v, g, beta = _seq(rng, n, T, d, d, GATE_SCALAR)
    S0 = rng.standard_normal((n, d, d))
    a = oracle.run(Params(d, d, mode=MODE_NAIVE), S0, q, k, v, g, beta)
    b = oracle.run(Params(d, d, window=1, n_comp_rows=0, n_comp_cols=0, smooth=0, mode=MODE_WINDOW),
                   S0, q, k, v, g, beta)
    np.testing.assert_array_equal(a.o, b.o)
    np.testing.assert_array_equal(a.Q, b.Q)
