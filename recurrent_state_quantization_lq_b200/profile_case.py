"""Run a short, fixed sequence of liblq launches for a profiler to capture.

    python -m recurrent_state_quantization_lq_b200.profile_case [--workload NAME]
        [--mode window|fp32|naive] [--tokens T] [--flush] [--prompt P] [--batch B]

Sets up one layer-state of the workload (prefill from a seeded FP32 state),
then runs T decode launches (the windowed kernel sees 0..T-1 buffered tokens)
and, with --flush, one window flush.  Launch order: the prefill's encode
launch (windowed/naive modes), then the T decode launches, then the flush.
With --prompt P the state is instead prefilled from a P-token prompt by one
token-prefill launch (lq_prefill_tokens).  --batch overrides the workload's
batch (smaller captures).  With --ragged-due S the handle is ragged: W - 1
decode launches with every sequence active, one with only the first S
sequences active (their windows are then full), then one flush of the due
units (the cluster flush); --tokens and --flush are ignored.
"""
from __future__ import annotations

import argparse

import torch

from recurrent_state_quantization_lq_b200 import inputs, lq


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="gdn_b64_h32_d128_w64", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--mode", default="window", choices=["window", "fp32", "naive"])
    ap.add_argument("--tokens", type=int, default=34)
    ap.add_argument("--flush", action="store_true")
    ap.add_argument("--prompt", type=int, default=0)
    ap.add_argument("--batch", type=int, default=0)
    ap.add_argument("--ragged-due", type=int, default=-1)
    args = ap.parse_args()
    wl = inputs.WORKLOADS[args.workload]
    if args.batch:
        wl = inputs.Workload(wl.name, args.batch, wl.heads, wl.d_k, wl.d_v, wl.window, wl.n_comp_rows,
                             wl.n_comp_cols, wl.per_channel_gate, wl.prefill_tokens, wl.decode_tokens, wl.dtype,
                             wl.seed, planted=wl.planted)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T = min(args.tokens, wl.window) if args.mode == "window" else args.tokens
    tb = inputs.tokens_on_device(wl.seed, T, wl.batch, wl.heads, wl.d_k, wl.d_v, wl.per_channel_gate, wl.dtype, dev)
    S0 = 0.3 * torch.randn(wl.batch, wl.heads, wl.d_v, wl.d_k, device=dev,
                           generator=torch.Generator(device=dev).manual_seed(wl.seed))
    ragged = args.ragged_due >= 0
    if ragged:
        T = wl.window
        tb = inputs.tokens_on_device(wl.seed, T, wl.batch, wl.heads, wl.d_k, wl.d_v, wl.per_channel_gate, wl.dtype,
                                     dev)
    st = lq.DecodeState(wl.batch, wl.heads, wl.d_k, window=wl.window, n_comp_rows=wl.n_comp_rows,
                        n_comp_cols=wl.n_comp_cols, gate="channel" if wl.per_channel_gate else "scalar",
                        mode=args.mode, in_dtype=wl.dtype, ragged=ragged, device=dev)
    if args.prompt:
        pb = inputs.tokens_on_device(wl.seed + 1, args.prompt, wl.batch, wl.heads, wl.d_k, wl.d_v,
                                     wl.per_channel_gate, wl.dtype, dev)
        po = torch.empty(args.prompt, wl.batch, wl.heads, wl.d_v, dtype=torch.float32, device=dev)
        st.prefill_tokens(pb.q, pb.k, pb.v, pb.g, pb.beta, S0=S0, out=po)
    else:
        st.prefill(S0)
    out = torch.empty(wl.batch, wl.heads, wl.d_v, dtype=torch.float32, device=dev)
    if ragged:
        act = torch.ones(wl.batch, dtype=torch.uint8, device=dev)
        for t in range(T):
            if t == T - 1:
                act[args.ragged_due:] = 0
            st.decode_step(tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t], out=out, active=act)
        st.flush()
    else:
        for t in range(T):
            st.decode_step(tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t], out=out)
        if args.flush:
            st.flush()
    status = st.device_status()
    if status != lq.LQ_OK:
        raise lq.LQError(status, "profile_case")
    print(f"profile_case: {wl.name} batch={wl.batch} mode={args.mode} prompt={args.prompt} tokens={T} "
          f"flush={args.flush} ragged_due={args.ragged_due} ok")


if __name__ == "__main__":
    main()
