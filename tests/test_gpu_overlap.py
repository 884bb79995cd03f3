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


@pytest.mark.parametrize("batch,window", [(37, 8), (40, 8), (2, 8)])
def test_ticket_counters_return_to_zero(batch, window):
    """The decode and the flush hand out units by ticket counters kept in the
    error region (int32 words 32-35).  Every launch starts from zero and the
    CTA that draws its last ticket sets the counter back, so both read zero
    after every decode and flush, whatever the grid; and a checkpoint taken
    between launches resumes on any number of SMs.  On 148 SMs (592 decode
    CTAs, 296 flush CTAs) 37 x 32 = 1184 units fill two whole decode rounds,
    40 x 32 leaves a partial one of 96, and 2 x 32 needs no ticket at all."""
    a, b = _pair(batch, 13, same=True)
    tb = inputs.tokens_on_device(7, 2 * window, batch, H, D, D, False, torch.bfloat16, DEV)
    zero = torch.zeros(4, dtype=torch.int32)
    for t in range(2 * window):
        oa = a.decode_step(*_tok(tb, t))
        assert torch.equal(a.view("err")[32:36].cpu(), zero), t
        assert torch.equal(oa, b.decode_step(*_tok(tb, t))), t
        if t % window == window - 1:
            a.flush()
            b.flush()
            assert torch.equal(a.view("err")[32:36].cpu(), zero), t
    assert a.device_status() == lq.LQ_OK and b.device_status() == lq.LQ_OK


def test_ticket_counter_left_set_is_reported():
    """A counter that is not zero when a launch starts (as a launch that ended
    on a device error may leave it) hands out tickets past the launch's range:
    the kernels report LQ_DEVERR_BOUNDS instead of going on silently, and a
    prefill clears the counters again."""
    batch = 40                                          # decode and flush both draw
    a, _ = _pair(batch, 14)
    tb = inputs.tokens_on_device(8, 2, batch, H, D, D, False, torch.bfloat16, DEV)
    big = torch.tensor([0, 1 << 20, 0, 1 << 20], dtype=torch.int32, device=DEV)
    a.view("err")[32:36].copy_(big)
    a.decode_step(*_tok(tb, 0))
    assert a.device_status() == lq.LQ_ERR_DEVICE
    err = a.view("err")[:3].cpu()
    assert int(err[0]) == lq.LQ_DEVERR_BOUNDS and int(err[2]) == -50
    a.prefill(None)
    assert torch.equal(a.view("err")[32:36].cpu(), torch.zeros(4, dtype=torch.int32))
    a.decode_step(*_tok(tb, 1))
    a.flush()
    assert a.device_status() == lq.LQ_OK
