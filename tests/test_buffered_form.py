"""Brute-force checks of the buffered form the CUDA decode uses (CPU only, FP64, tiny heads).

Within a window that starts from the decoded state S~ = R^ + C, with
G_t = sum of the log-gates since the window start and gamma_t = exp(G_t):
  S_t = S~ diag(gamma_t) + sum_{j<=t} delta_j (kappa_j * gamma_t)^T,
  kappa_j = k_j / gamma_j,  delta_j = beta_j (v_j - S_{j-1}(alpha_j * k_j)),
so a decode step needs only one pass over the fixed INT8 state plus the
buffered (delta_j, kappa_j) pairs; compensators are buffered pairs with G = 0
(LeapQuant, "Abstract (arXiv)": Compensator Tokens take the same update path
as real tokens).  The WY form writes the same product of transitions as
Gamma_t - sum_j w_j (k_j * gamma_t / gamma_j)^T, and delta_t = v~_t - S~ u_t.
These are checked against the oracle's dense recurrence and against explicit
products of the transition matrices.
"""
import numpy as np
import pytest

import oracle
from oracle import GATE_CHANNEL, GATE_SCALAR, MODE_FP32, MODE_WINDOW, Params


def _unit(rng, d):
    x = rng.standard_normal(d)
    return x / np.linalg.norm(x)


def _window_inputs(rng, W, dk, dv, gate):
    q = np.stack([_unit(rng, dk) for _ in range(W)])
    k = np.stack([_unit(rng, dk) for _ in range(W)])
    v = rng.standard_normal((W, dv))
    g = -rng.uniform(0.01, 0.4, (W, 1 if gate == GATE_SCALAR else dk))
    beta = rng.uniform(0.05, 0.95, W)
    return q, k, v, g, beta


def _buffered_window(enc, dk, dv, q, k, v, g, beta):
    """Outputs of one window and the rebuilt end state, from the encoded
    window-start state and the buffered pairs only (never a dense S_t)."""
    R_hat = enc.sigma.astype(np.float64)[:, None] * enc.Q * enc.s.astype(np.float64)[None, :]
    deltas, kappas = [], []
    for c, i in enumerate(enc.comp_rows):          # row compensator: (e_i, k_c)
        e = np.zeros(dv); e[i] = 1.0
        deltas.append(e); kappas.append(enc.row_vecs[c].astype(np.float64))
    for c, j in enumerate(enc.comp_cols):          # column compensator: (v_c, e_j)
        e = np.zeros(dk); e[j] = 1.0
        deltas.append(enc.col_vecs[c].astype(np.float64)); kappas.append(e)
    G = np.zeros(dk)
    outs = []
    for t in range(len(beta)):
        G = G + g[t]
        gam = np.exp(G)
        xk, xq = gam * k[t], gam * q[t]
        Sk = R_hat @ xk + sum(d * (kap @ xk) for d, kap in zip(deltas, kappas))
        delta = beta[t] * (v[t] - Sk)
        o = R_hat @ xq + sum(d * (kap @ xq) for d, kap in zip(deltas, kappas)) + delta * (k[t] @ q[t])
        outs.append(o)
        deltas.append(delta); kappas.append(k[t] / gam)
    gam = np.exp(G)
    S_end = R_hat * gam[None, :] + sum(np.outer(d, kap * gam) for d, kap in zip(deltas, kappas))
    return np.array(outs), S_end


@pytest.mark.parametrize("gate", [GATE_SCALAR, GATE_CHANNEL])
@pytest.mark.parametrize("dims", [(4, 4, 1, 1), (8, 6, 2, 1), (8, 8, 0, 0)])
def test_buffered_form_matches_dense_oracle(gate, dims):
    dk, dv, nr, nc = dims
    rng = np.random.default_rng(20 + dk + nr)
    for W in (1, 3, 8):
        S0 = rng.standard_normal((dv, dk)) * 3
        S0[rng.integers(dv)] *= 20
        q, k, v, g, beta = _window_inputs(rng, W, dk, dv, gate)
        p = Params(dk, dv, window=W, n_comp_rows=nr, n_comp_cols=nc, gate=gate, mode=MODE_WINDOW)
        enc = oracle.encode(p, S0)
        dense = oracle.run(p, S0[None], q[None], k[None], v[None], g[None], beta[None])
        o_buf, S_end = _buffered_window(enc, dk, dv, q, k, v, g, beta)
        np.testing.assert_allclose(o_buf, dense.o[0], rtol=0, atol=1e-12)
        # end state before the flush encodes it: the unquantized recurrence from S~
        plain = oracle.run(Params(dk, dv, gate=gate, mode=MODE_FP32), enc.S_tilde[None], q[None],
                           k[None], v[None], g[None], beta[None])
        np.testing.assert_allclose(S_end, plain.S_final[0], rtol=0, atol=1e-12)


@pytest.mark.parametrize("gate", [GATE_SCALAR, GATE_CHANNEL])
def test_wy_form_against_explicit_products(gate):
    dk, dv, W = 6, 5, 7
    rng = np.random.default_rng(30)
    q, k, v, g, beta = _window_inputs(rng, W, dk, dv, gate)
    S_tilde = rng.standard_normal((dv, dk))
    p = Params(dk, dv, gate=gate, mode=MODE_FP32)
    # explicit transition matrices A_t = diag(alpha_t)(I - beta_t k_t k_t^T)
    A = [np.diag(np.exp(g[t]) * np.ones(dk)) @ (np.eye(dk) - beta[t] * np.outer(k[t], k[t]))
         for t in range(W)]
    # WY recursion: w_t = beta_t (gamma_t*k_t - sum_{j<t} w_j ((k_j/gamma_j).(gamma_t*k_t)))
    G = np.cumsum(g, axis=0) * np.ones((W, dk))
    gam = np.exp(G)
    w, vt = [], []
    S = S_tilde.copy()
    for t in range(W):
        x = gam[t] * k[t]
        w_t = beta[t] * (x - sum(w[j] * ((k[j] / gam[j]) @ x) for j in range(t)))
        v_t = beta[t] * (v[t] - sum(vt[j] * ((k[j] / gam[j]) @ x) for j in range(t)))
        w.append(w_t); vt.append(v_t)
        P = np.eye(dk)
        for j in range(t + 1):
            P = P @ A[j]
        P_wy = np.diag(gam[t]) - sum(np.outer(w[j], k[j] * gam[t] / gam[j]) for j in range(t + 1))
        np.testing.assert_allclose(P_wy, P, atol=1e-12)
        # delta_t from the dense oracle state equals v~_t - S~ u_t (u_t = w_t)
        delta_dense = beta[t] * (v[t] - S @ (np.exp(g[t]) * np.ones(dk) * k[t]))
        np.testing.assert_allclose(delta_dense, v_t - S_tilde @ w_t, atol=1e-12)
        S, _ = oracle.step(p, S, q[t], k[t], v[t], g[t], beta[t])
