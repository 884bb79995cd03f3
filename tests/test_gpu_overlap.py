"""The windowed decode kernel starts while the kernel before it in the stream
finishes (programmatic dependent launch).  These cases put a kernel that writes
what the decode reads directly before it, with no synchronization between the
two: the decode's outputs must equal those of a decode that did not overlap.
Both the mma.sync pass (64 units) and the tcgen05 pass (1216 units) run.
"""
import pytest
import torch

from recurrent_state_quantization_lq_b200 import inputs, lq

pytestmark = pytest.mark.gpu
DEV = "cuda"
H, D, W = 32, 128, 8


def _pair(batch, seed, same=False):
    """Two windowed states over different (or, with same, equal) random states."""
    gen = torch.Generator().manual_seed(seed)
    S = [(0.5 * torch.randn(batch, H, D, D, generator=gen)).to(DEV) for _ in range(2)]
    if same:
        S[1] = S[0].clone()
    st = [lq.DecodeState(batch, H, D, window=W, device=DEV) for _ in range(2)]
    for s, S0 in zip(st, S):
        s.prefill(S0)
    return st


def _tok(tb, t):
    return tb.q[t], tb.k[t], tb.v[t], tb.g[t], tb.beta[t]


@pytest.mark.parametrize("batch", [2, 38])
def test_codes_rewritten_by_a_kernel_then_resume(batch):
    """State a's workspace is overwritten with state b's by an elementwise
    kernel right before a's decode; lq_state_resume tells the handle, so the
    decode must read b's codes, not the ones a's earlier decodes settled."""
    a, b = _pair(batch, 11)
    tb = inputs.tokens_on_device(5, W, batch, H, D, D, False, torch.bfloat16, DEV)
    for t in range(3):
        a.decode_step(*_tok(tb, t))
        b.decode_step(*_tok(tb, t))
    torch.add(b.workspace, 0, out=a.workspace)          # a kernel, on the same stream
    assert lq.lib().lq_state_resume(a._h, 3) == lq.LQ_OK
    for t in range(3, 6):                               # the first after resume, then settled ones
        oa = a.decode_step(*_tok(tb, t))
        ob = b.decode_step(*_tok(tb, t))
        assert torch.equal(oa, ob), t
    assert a.device_status() == lq.LQ_OK and b.device_status() == lq.LQ_OK


@pytest.mark.parametrize("batch", [2, 38])
def test_inputs_written_by_the_previous_kernel(batch):
    """Each step's q, k, v, g, beta are produced by a kernel launched just
    before the decode into buffers that held NaN: a decode that read them
    before that kernel completed would see NaN."""
    a, b = _pair(batch, 12, same=True)
    tb = inputs.tokens_on_device(6, W, batch, H, D, D, False, torch.bfloat16, DEV)
    bufs = [torch.full_like(x[0], float("nan")) for x in (tb.q, tb.k, tb.v, tb.g, tb.beta)]
    for t in range(W):
        src = _tok(tb, t)
        ob = b.decode_step(*src)
        for dst, x in zip(bufs, src):
            torch.mul(x, 1, out=dst)
        oa = a.decode_step(*bufs)
        assert torch.equal(oa, ob), t
        for dst in bufs:
            dst.fill_(float("nan"))
    a.flush()
    b.flush()
    src = _tok(tb, 0)
    for dst, x in zip(bufs, src):
        torch.mul(x, 1, out=dst)
    assert torch.equal(a.decode_step(*bufs), b.decode_step(*src))
    assert a.device_status() == lq.LQ_OK and b.device_status() == lq.LQ_OK
