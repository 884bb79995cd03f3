"""Helpers for the parity tests: drive the CUDA path through the C-ABI binding
and the oracle on the same seeded inputs, and compare them."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from recurrent_state_quantization_lq_b200 import inputs, lq

MODES = {"window": oracle.MODE_WINDOW, "naive": oracle.MODE_NAIVE, "fp32": oracle.MODE_FP32}


def oracle_params(d, window=64, nr=2, nc=2, gate="scalar", mode="window", smooth=1, select="l2"):
    return oracle.Params(d_k=d, d_v=d, window=window, n_comp_rows=nr, n_comp_cols=nc,
                         gate=oracle.GATE_SCALAR if gate == "scalar" else oracle.GATE_CHANNEL,
                         mode=MODES[mode], smooth=smooth,
                         select=oracle.SELECT_L2 if select == "l2" else oracle.SELECT_MAXABS)


def unit_inputs(tb: inputs.TokenBatch, units) -> tuple:
    """Oracle arrays (FP64, head-major) of the given flattened units."""
    T, B, H = tb.q.shape[:3]
    units = list(units)

    def pick(x):
        x = x.reshape(T, B * H, *x.shape[3:])[:, units]
        return x.transpose(0, 1).double().numpy()

    return pick(tb.q), pick(tb.k), pick(tb.v), pick(tb.g), pick(tb.beta)


def snapshot(st: lq.DecodeState) -> dict:
    """The encoded window-start state, read through lq_state_export (absent
    regions are None)."""
    names = ("codes", "row_scale", "col_smooth", "comp_index", "comp_row_vec", "comp_col_vec")
    shapes = st.export_shapes()
    got = st.export([n for n in names if n in shapes])
    return {n: got.get(n) for n in names}


def to_device(tb: inputs.TokenBatch, device) -> inputs.TokenBatch:
    return inputs.TokenBatch(*(x.to(device) for x in (tb.q, tb.k, tb.v, tb.g, tb.beta)))


def gpu_run(st: lq.DecodeState, tb_dev: inputs.TokenBatch, flush_every: int | None = None,
            flush_at_end: bool = False, snaps: bool = True):
    """Decode every token of tb_dev; flush after every `flush_every` tokens.
    Returns (outputs [T,B,H,d] CPU FP32, list of snapshots after each flush)."""
    T = tb_dev.q.shape[0]
    outs = torch.empty((T, st.batch, st.heads, st.d), dtype=torch.float32, device=st.device)
    shots = []
    for t in range(T):
        st.decode_step(tb_dev.q[t], tb_dev.k[t], tb_dev.v[t], tb_dev.g[t], tb_dev.beta[t], out=outs[t])
        if flush_every and (t + 1) % flush_every == 0:
            st.flush()
            if snaps:
                shots.append(snapshot(st))
    if flush_at_end and st.fill > 0:
        st.flush()
        if snaps:
            shots.append(snapshot(st))
    torch.cuda.synchronize()
    return outs.cpu(), shots


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def compare_codes(q_gpu: np.ndarray, q_ref: np.ndarray) -> tuple[float, int]:
    """(fraction of equal codes, largest code difference)."""
    d = np.abs(q_gpu.astype(np.int32) - q_ref.astype(np.int32))
    return float((d == 0).mean()), int(d.max()) if d.size else 0


def import_encoded(st: lq.DecodeState, ref: oracle.RunResult, f: int, units=None) -> None:
    """Write the oracle's f-th encoded state into the GPU workspace (all units,
    or the listed flattened units).  The window buffer must be empty."""
    B, H, d = st.batch, st.heads, st.d
    units = list(range(B * H)) if units is None else list(units)
    sel = torch.tensor(units, dtype=torch.long)
    dev = st.device

    def put(name, arr):
        v = st.view(name)
        flat = v.view(B * H, *v.shape[2:])
        flat[sel.to(dev)] = torch.as_tensor(np.ascontiguousarray(arr)).to(dev, flat.dtype).reshape(
            len(units), *flat.shape[1:])

    put("codes", ref.Q[:, f])
    put("row_scale", ref.sigma[:, f])
    if "col_smooth" in st.export_shapes():
        put("col_smooth", ref.s[:, f])
    nr, nc = st.cfg.n_comp_rows, st.cfg.n_comp_cols
    if st.cfg.mode == 0 and nr + nc > 0:
        idx = np.zeros((len(units), st.layout.comp_index_stride), np.int32)
        idx[:, :nr + nc] = ref.idx[:, f]
        put("comp_index", idx)
        if nr:
            put("comp_row_vec", ref.vec[:, f, :nr * d].reshape(len(units), nr, d))
        if nc:
            put("comp_col_vec", ref.vec[:, f, nr * d:].reshape(len(units), nc, d))
    torch.cuda.synchronize()


def decoded_state(ref: oracle.RunResult, f: int, nr: int, nc: int, d: int) -> np.ndarray:
    """S~ = sigma Q s + C of the oracle's f-th encoding, [n, d, d] FP64."""
    S = ref.sigma[:, f].astype(np.float64)[:, :, None] * ref.Q[:, f] * ref.s[:, f].astype(np.float64)[:, None, :]
    for n in range(S.shape[0]):
        for c in range(nr):
            S[n, ref.idx[n, f, c], :] += ref.vec[n, f, c * d:(c + 1) * d]
        for c in range(nc):
            S[n, :, ref.idx[n, f, nr + c]] += ref.vec[n, f, nr * d + c * d:nr * d + (c + 1) * d]
    return S


def selection_is_near_tie(S_pre: np.ndarray, got_idx, ref_idx, nr: int, select: str = "l2",
                          rtol: float = 1e-5) -> bool:
    """Both compensator selections rank equally well on the oracle's FP32
    pre-flush state up to rtol (a legitimate alternative at a near-tie)."""
    R = S_pre.astype(np.float32).astype(np.float64)
    def score(M, axis):
        return (M ** 2).sum(axis=axis) if select == "l2" else np.abs(M).max(axis=axis)
    rows = score(R, 1)
    g_rows, r_rows = list(got_idx[:nr]), list(ref_idx[:nr])
    if not np.allclose(np.sort(rows[g_rows]), np.sort(rows[r_rows]), rtol=rtol, atol=0):
        return False
    Rz = R.copy()
    Rz[r_rows, :] = 0.0
    cols = score(Rz, 0)
    g_cols, r_cols = list(got_idx[nr:]), list(ref_idx[nr:])
    return bool(np.allclose(np.sort(cols[g_cols]), np.sort(cols[r_cols]), rtol=rtol, atol=0))
