"""The N > 1 path on CPU: two gloo ranks, each with its own shard of sequences.

The sharded decode has no data-path exchange, so what N processes add is host
plumbing: rank discovery, per-rank seeds, the barrier and the max over ranks of
the timer, and the whole-job rate.  These tests run that plumbing as two real
processes over gloo, and check that sharding the batch across ranks changes no
result: every rank's outputs and window-end codes (computed by the oracle on
its shard) equal the matching slice of one run over all ranks' sequences
together.
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from recurrent_state_quantization_lq_b200 import inputs, ranks

WORLD = 2
B_PER_RANK, H, D, T, W = 2, 2, 16, 12, 4
BASE_SEED = 5


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _params() -> oracle.Params:
    return oracle.Params(D, D, window=W, n_comp_rows=1, n_comp_cols=1)


def _shard_inputs(rank: int):
    """Rank `rank`'s seeded shard: tokens of B_PER_RANK sequences and their start states."""
    seed = ranks.shard_seed(BASE_SEED, rank)
    tb = inputs.tokens(seed, 0, T, B_PER_RANK, H, D, D, False, torch.float32)
    S0 = torch.randn(B_PER_RANK * H, D, D, generator=torch.Generator().manual_seed(seed),
                     dtype=torch.float64).numpy()
    return tb, S0


def _head_major(tb: inputs.TokenBatch):
    n = tb.q.shape[1] * tb.q.shape[2]

    def hm(x):
        return x.reshape(T, n, *x.shape[3:]).transpose(0, 1).double().numpy()

    return hm(tb.q), hm(tb.k), hm(tb.v), hm(tb.g), hm(tb.beta)


def _worker(rank: int, port: int, out_dir: str) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    ranks.init("gloo", timeout_s=60)
    try:
        assert ranks.env_ranks() == (rank, WORLD, rank)
        # the timer reduction: every rank must see the slowest rank's time
        t = 0.25 + rank
        assert ranks.max_over_ranks(t, WORLD) == 0.25 + WORLD - 1
        tb, S0 = _shard_inputs(rank)
        res = oracle.run(_params(), S0, *_head_major(tb), n_threads=1)
        ranks.barrier(WORLD)
        gathered = [None] * WORLD
        dist.all_gather_object(gathered, {"rank": rank, "o": res.o, "Q": res.Q,
                                          "q_sum": float(tb.q.double().sum())})
        if rank == 0:
            np.save(os.path.join(out_dir, "o.npy"), np.stack([g["o"] for g in gathered]))
            np.save(os.path.join(out_dir, "Q.npy"), np.stack([g["Q"] for g in gathered]))
            np.save(os.path.join(out_dir, "q_sum.npy"), np.array([g["q_sum"] for g in gathered]))
        ranks.barrier(WORLD)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def gathered(tmp_path_factory):
    out = tmp_path_factory.mktemp("multirank")
    mp.start_processes(_worker, args=(_free_port(), str(out)), nprocs=WORLD, join=True, start_method="spawn")
    return (np.load(out / "o.npy"), np.load(out / "Q.npy"), np.load(out / "q_sum.npy"))


def test_shards_are_distinct(gathered):
    _, _, q_sum = gathered
    assert len(set(q_sum.tolist())) == WORLD


def test_sharded_results_equal_one_job(gathered):
    o, Q, _ = gathered
    shards = [_shard_inputs(r) for r in range(WORLD)]
    # one job holding every rank's sequences, in rank order
    cat = [np.concatenate(parts) for parts in zip(*(_head_major(tb) for tb, _ in shards))]
    S0 = np.concatenate([s for _, s in shards])
    whole = oracle.run(_params(), S0, *cat, n_threads=1)
    n = B_PER_RANK * H
    for r in range(WORLD):
        np.testing.assert_array_equal(o[r], whole.o[r * n:(r + 1) * n])
        np.testing.assert_array_equal(Q[r], whole.Q[r * n:(r + 1) * n])


def test_shard_seeds():
    assert ranks.shard_seed(1, 0) != ranks.shard_seed(1, 1)
    assert ranks.shard_seed(1, 3) == ranks.shard_seed(1, 3)
    with pytest.raises(ValueError):
        ranks.shard_seed(1, 1000)


def test_whole_job_rate():
    # weak scaling: 2 ranks x 100 units in 0.5 s of the slowest rank
    assert ranks.whole_job_rate(100, 2, 0.5) == 400.0
    with pytest.raises(ValueError):
        ranks.whole_job_rate(100, 2, 0.0)


def test_single_process_defaults(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert ranks.env_ranks() == (0, 1, 0)
    assert ranks.max_over_ranks(3.5, 1) == 3.5
    ranks.barrier(1)
