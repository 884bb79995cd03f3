"""Seeded synthetic inputs for gated delta-rule decode.

This module only draws random numbers and shapes them into the input
distributions of the workloads; it holds none of the method's arithmetic, so
both the CUDA path and the CPU oracle can be fed from it.

Recipe (per token t of a sequence of P prefill + T decode tokens; every
(sequence, head) pair is an independent recurrence):
  q, k ~ N(0, 1)^d, each L2-normalised over its d channels in FP32;
  v ~ N(0, 1)^d_v;  beta = sigmoid(N(0, 1));
  g = log(alpha) = -0.1 * softplus(N(0, 1)), one draw per head (scalar gate)
      or one per key channel (per-channel gate), so alpha ~ 0.92 on average.
q, k, v are then cast to the input dtype (bf16 or FP32); g and beta stay FP32.
Token t draws from its own generator, seeded from (seed, t), so any token
range can be produced without drawing the tokens before it.

Initial states: zeros, or N(0, 1) with planted outlier rows and columns: per
(sequence, head), `n_rows` rows and `n_cols` columns are drawn without
replacement and every entry lying in a planted row or column is multiplied
by `scale` once (an entry in both is scaled once, not twice).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

_TOKEN_MIX = 1_000_003
_STATE_MIX = 7_919


def _gen(seed: int, t: int, stream: int = 0) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((seed * _TOKEN_MIX + t) * 31 + stream)
    return g


@dataclass
class TokenBatch:
    """Inputs of tokens [t0, t1) for all (sequence, head) pairs.

    q, k: [T, B, H, d_k]; v: [T, B, H, d_v] in the input dtype;
    g: [T, B, H] (scalar gate) or [T, B, H, d_k] (per-channel gate), FP32;
    beta: [T, B, H], FP32.
    """
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor


def tokens(seed: int, t0: int, t1: int, batch: int, heads: int, d_k: int, d_v: int,
           per_channel_gate: bool, dtype: torch.dtype = torch.bfloat16) -> TokenBatch:
    """Draw tokens [t0, t1) on the CPU (see the module docstring for the recipe)."""
    T = t1 - t0
    q = torch.empty(T, batch, heads, d_k, dtype=dtype)
    k = torch.empty(T, batch, heads, d_k, dtype=dtype)
    v = torch.empty(T, batch, heads, d_v, dtype=dtype)
    gshape = (batch, heads, d_k) if per_channel_gate else (batch, heads)
    g = torch.empty((T,) + gshape, dtype=torch.float32)
    beta = torch.empty(T, batch, heads, dtype=torch.float32)
    for i, t in enumerate(range(t0, t1)):
        gen = _gen(seed, t)
        qt = torch.randn(batch, heads, d_k, generator=gen)
        kt = torch.randn(batch, heads, d_k, generator=gen)
        vt = torch.randn(batch, heads, d_v, generator=gen)
        bt = torch.randn(batch, heads, generator=gen)
        gt = torch.randn(gshape, generator=gen)
        q[i] = (qt / qt.norm(dim=-1, keepdim=True)).to(dtype)
        k[i] = (kt / kt.norm(dim=-1, keepdim=True)).to(dtype)
        v[i] = vt.to(dtype)
        beta[i] = torch.sigmoid(bt)
        g[i] = -0.1 * torch.nn.functional.softplus(gt)
    return TokenBatch(q, k, v, g, beta)


def planted_state(seed: int, batch: int, heads: int, d_v: int, d_k: int,
                  n_rows: int = 2, n_cols: int = 2, scale: float = 50.0):
    """N(0,1) states [B, H, d_v, d_k] with planted outlier rows/columns.

    Returns (S0 FP32, rows int64 [B, H, n_rows], cols int64 [B, H, n_cols]).
    """
    gen = _gen(seed, 0, stream=_STATE_MIX)
    S = torch.randn(batch, heads, d_v, d_k, generator=gen)
    rows = torch.empty(batch, heads, n_rows, dtype=torch.int64)
    cols = torch.empty(batch, heads, n_cols, dtype=torch.int64)
    for b in range(batch):
        for h in range(heads):
            rows[b, h] = torch.randperm(d_v, generator=gen)[:n_rows]
            cols[b, h] = torch.randperm(d_k, generator=gen)[:n_cols]
    mask = torch.zeros(batch, heads, d_v, d_k, dtype=torch.bool)
    bi = torch.arange(batch)[:, None, None]
    hi = torch.arange(heads)[None, :, None]
    mask[bi, hi, rows, :] = True
    mask.transpose(-1, -2)[bi, hi, cols, :] = True
    S = torch.where(mask, S * scale, S)
    return S, rows, cols


@dataclass(frozen=True)
class Workload:
    """A named decode workload (sizes and recipe, no arithmetic)."""
    name: str
    batch: int
    heads: int
    d_k: int
    d_v: int
    window: int
    n_comp_rows: int
    n_comp_cols: int
    per_channel_gate: bool
    prefill_tokens: int
    decode_tokens: int
    dtype: torch.dtype
    seed: int
    planted: bool = False
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def units(self) -> int:
        return self.batch * self.heads


WORKLOADS = {
    # tiny GDN check: 1 sequence, 1 head, 64x64 state from zero, W=64, 2+2 compensators, FP32 in
    "gdn_tiny_d64": Workload("gdn_tiny_d64", 1, 1, 64, 64, 64, 2, 2, False, 0, 256, torch.float32, 0),
    # GDN decode: 64 sequences x 32 heads, 128x128 state after a 512-token FP32 prefill, W=64, n_c=4
    "gdn_b64_h32_d128_w64": Workload("gdn_b64_h32_d128_w64", 64, 32, 128, 128, 64, 2, 2, False,
                                     512, 1024, torch.bfloat16, 1),
    # KDA-style decode: per-key-channel gate, 128 sequences, W=128, n_c=8
    "kda_b128_h32_d128_w128": Workload("kda_b128_h32_d128_w128", 128, 32, 128, 128, 128, 4, 4, True,
                                       512, 1024, torch.bfloat16, 2),
    # outlier stress: N(0,1) state with 2 planted rows + 2 planted columns x50, 4096 tokens, W=64
    "gdn_outlier_b256_h32_d128_w64": Workload("gdn_outlier_b256_h32_d128_w64", 256, 32, 128, 128, 64,
                                              2, 2, False, 0, 4096, torch.bfloat16, 3, planted=True),
}


def sweep_workload(batch: int, window: int) -> Workload:
    """One point of the GDN batch x window sweep (32 heads, 128x128, 2048 tokens, n_c=4)."""
    return Workload(f"gdn_sweep_b{batch}_w{window}", batch, 32, 128, 128, window, 2, 2, False,
                    512, 2048, torch.bfloat16, 4)


def tokens_on_device(seed: int, T: int, batch: int, heads: int, d_k: int, d_v: int,
                     per_channel_gate: bool, dtype: torch.dtype, device,
                     chunk: int = 64) -> TokenBatch:
    """The same recipe drawn on the GPU from a CUDA generator (for timing runs
    that need gigabytes of tokens; its stream differs from `tokens`)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed * _TOKEN_MIX + 17)
    q = torch.empty(T, batch, heads, d_k, dtype=dtype, device=device)
    k = torch.empty_like(q)
    v = torch.empty(T, batch, heads, d_v, dtype=dtype, device=device)
    gshape = (batch, heads, d_k) if per_channel_gate else (batch, heads)
    g = torch.empty((T,) + gshape, dtype=torch.float32, device=device)
    beta = torch.empty(T, batch, heads, dtype=torch.float32, device=device)
    for t0 in range(0, T, chunk):
        n = min(chunk, T - t0)
        x = torch.randn(n, batch, heads, d_k, generator=gen, device=device)
        q[t0:t0 + n] = (x / x.norm(dim=-1, keepdim=True)).to(dtype)
        x = torch.randn(n, batch, heads, d_k, generator=gen, device=device)
        k[t0:t0 + n] = (x / x.norm(dim=-1, keepdim=True)).to(dtype)
        v[t0:t0 + n] = torch.randn(n, batch, heads, d_v, generator=gen, device=device).to(dtype)
        beta[t0:t0 + n] = torch.sigmoid(torch.randn(n, batch, heads, generator=gen, device=device))
        g[t0:t0 + n] = -0.1 * torch.nn.functional.softplus(
            torch.randn((n,) + gshape, generator=gen, device=device))
    return TokenBatch(q, k, v, g, beta)
