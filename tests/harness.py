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
    out = {}
    for name in ("codes", "row_scale", "col_smooth", "comp_index", "comp_row_vec", "comp_col_vec"):
        v = st.view(name)
        out[name] = None if v is None else v.detach().cpu().clone()
    return out


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
