"""The tensor-core INT8 pass of the windowed decode against the oracle.

For d = 128 the launcher runs the INT8 pass on tcgen05 once the CTAs walk two
units or more each, and on warp-level MMA below that; the other parity tests
are small enough to take the warp-level pass.  These cases use enough units
for the tensor-core pass, for every gate, input type and window-phase kind,
and check a seeded sample of units against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from harness import compare_codes, gpu_run, oracle_params, rel_l2, to_device, unit_inputs
from recurrent_state_quantization_lq_b200 import inputs, lq
from test_gpu_ragged import _ragged_case

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
H, D = 32, 128


def _batch() -> int:
    """Sequences for more than two units per CTA at 4 CTAs per SM."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return -(-8 * sms // H) + 1


@pytest.mark.parametrize("gate", ["scalar", "channel"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_tensor_core_pass_shared_phase(gate, dtype):
    B, W = _batch(), 8
    T = 2 * W + 3
    tb = inputs.tokens(61, 0, T, B, H, D, D, gate == "channel", dtype)
    S0 = 0.5 * torch.randn(B, H, D, D, generator=torch.Generator().manual_seed(61))
    st = lq.DecodeState(B, H, D, window=W, n_comp_rows=2, n_comp_cols=2, gate=gate, in_dtype=dtype, device=DEV)
    st.prefill(S0.to(DEV).contiguous())
    o_gpu, shots = gpu_run(st, to_device(tb, DEV), flush_every=W)
    assert st.device_status() == lq.LQ_OK
    assert torch.isfinite(o_gpu).all()

    units = sorted(np.random.default_rng(61).choice(B * H, 6, replace=False).tolist())
    ref = oracle.run(oracle_params(D, W, 2, 2, gate), S0.reshape(B * H, D, D)[units].double().numpy(),
                     *unit_inputs(tb, units))
    o_s = o_gpu.reshape(T, B * H, D)[:, units].transpose(0, 1).numpy()
    err = rel_l2(o_s, ref.o)
    assert err <= 1e-3, err
    frac, worst = compare_codes(shots[0]["codes"].reshape(B * H, D, D)[units].numpy(), ref.Q[:, 1])
    assert frac >= 0.999 and worst <= 1, (frac, worst)


@pytest.mark.parametrize("gate,dtype", [("scalar", torch.bfloat16), ("channel", torch.float32)])
def test_tensor_core_pass_ragged_phases(gate, dtype):
    B = _batch()
    rng = np.random.default_rng(62)
    sample = list(zip(rng.choice(B, 6, replace=False).tolist(), rng.choice(H, 6).tolist()))
    _ragged_case(D, gate, dtype, W=8, nr=2, nc=2, B=B, H=H, T=24, seed=62, p_active=0.9, sample=sample)
