"""The seeded input generator (CPU only): shapes, recipe and determinism."""
import torch

from recurrent_state_quantization_lq_b200 import inputs


def test_token_ranges_are_consistent_and_deterministic():
    a = inputs.tokens(5, 0, 6, 2, 3, 16, 8, per_channel_gate=True)
    b = inputs.tokens(5, 2, 5, 2, 3, 16, 8, per_channel_gate=True)
    for x, y in zip((a.q, a.k, a.v, a.g, a.beta), (b.q, b.k, b.v, b.g, b.beta)):
        assert torch.equal(x[2:5], y)
    assert a.q.dtype == torch.bfloat16 and a.g.dtype == torch.float32
    assert a.g.shape == (6, 2, 3, 16) and a.beta.shape == (6, 2, 3)


def test_recipe_ranges():
    tb = inputs.tokens(0, 0, 64, 4, 4, 64, 64, per_channel_gate=False, dtype=torch.float32)
    n = tb.q.norm(dim=-1)
    assert torch.allclose(n, torch.ones_like(n), atol=1e-5)
    assert (tb.beta > 0).all() and (tb.beta < 1).all()
    alpha = tb.g.exp()
    assert (alpha < 1).all() and (alpha > 0.5).all()
    assert 0.90 < alpha.mean().item() < 0.95


def test_planted_state_scales_rows_and_columns_once():
    S, rows, cols = inputs.planted_state(1, 2, 2, 32, 16, scale=50.0)
    torch.manual_seed(0)
    for b in range(2):
        for h in range(2):
            r, c = rows[b, h].tolist(), cols[b, h].tolist()
            assert len(set(r)) == 2 and len(set(c)) == 2
            mask = torch.zeros(32, 16, dtype=torch.bool)
            mask[r, :] = True
            mask[:, c] = True
            big = S[b, h].abs()
            # planted entries are N(0,1)*50 and the rest N(0,1): compare typical sizes
            assert big[mask].median() > 20 * big[~mask].median()
            assert big[mask].median() < 80 * big[~mask].median()   # x50 once, not x2500
