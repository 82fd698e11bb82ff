"""Multi-rank host logic of bench.py, on CPU with two gloo ranks.

The decode path shards by sequence with no exchange: each rank owns a batch
(its own pool, block tables and sequences) and the only collectives are the
barrier and the reduction of the timing figures. These tests run that host
logic with world_size 2 on the gloo backend: the per-rank seeds give different
batches, each rank's batch decodes through the oracle, and the whole-job
figures are the sum of the units over ranks divided by the slowest rank's time.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
import workloads

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = workloads.CONFIGS["tiny"]
        b = workloads.make_batch("tiny", seed=bench.rank_seed(cfg.seed, rank), device="cpu", poison=True)
        out = oracle.decode_step(b)[0]
        kv = workloads.kv_bytes(b)
        S = b.num_seqs
        tok = int(b.context_lens.sum())
        total_ms = 10.0 * (rank + 1)            # rank 1 is the slower one
        job = bench.job_totals(kv, S, tok, 3, total_ms)
        sums, maxes = bench.aggregate([float(rank + 1), 2.0], [float(rank), -float(rank)])
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), out=out, kv=kv, S=S, tok=tok,
                 value=job["value"], seq=job["seq_per_s"], toks=job["ctx_tokens_per_s"], max_ms=job["max_ms"],
                 sums=np.array(sums), maxes=np.array(maxes),
                 lens=b.context_lens.numpy(), q=b.q.float().numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def ranks(tmp_path_factory):
    d = tmp_path_factory.mktemp("gloo")
    mp.start_processes(_worker, args=(WORLD, _free_port(), str(d)), nprocs=WORLD, join=True, start_method="spawn")
    return [dict(np.load(d / f"rank{r}.npz")) for r in range(WORLD)]


def test_aggregate_sums_and_maxes_over_ranks(ranks):
    for r in ranks:
        assert r["sums"].tolist() == [3.0, 4.0]
        assert r["maxes"].tolist() == [1.0, 0.0]


def test_job_totals_are_sum_of_units_over_slowest_rank(ranks):
    kv = sum(int(r["kv"]) for r in ranks)
    seqs = sum(int(r["S"]) for r in ranks)
    toks = sum(int(r["tok"]) for r in ranks)
    seconds = 20.0 / 1e3                      # the slower rank's 20 ms
    for r in ranks:
        assert float(r["max_ms"]) == 20.0
        assert float(r["value"]) == pytest.approx(3 * kv / seconds / 1e9, rel=1e-12)
        assert float(r["seq"]) == pytest.approx(3 * seqs / seconds, rel=1e-12)
        assert float(r["toks"]) == pytest.approx(3 * toks / seconds, rel=1e-12)


def test_ranks_decode_different_batches_of_the_same_recipe(ranks):
    a, b = ranks
    assert a["q"].shape == b["q"].shape
    assert not np.array_equal(a["q"], b["q"])
    for r in ranks:
        assert np.isfinite(r["out"]).all()    # poisoned slots are never read


def test_rank_zero_uses_the_canonical_seed(ranks):
    b = workloads.make_batch("tiny", device="cpu", poison=True)
    assert np.array_equal(ranks[0]["q"], b.q.float().numpy())
    np.testing.assert_array_equal(ranks[0]["out"], oracle.decode_step(b)[0])


def test_job_totals_without_a_process_group_is_the_single_rank_figure():
    job = bench.job_totals(1e9, 10, 1000, 4, 2000.0)
    assert job == {"value": 2.0, "seq_per_s": 20.0, "ctx_tokens_per_s": 2000.0, "max_ms": 2000.0}


def test_reference_arm_on_a_nonzero_rank_exits_without_work(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    def boom(*a, **k):
        raise AssertionError("rank 1 must not run the oracle")
    monkeypatch.setattr(bench, "run_reference", boom)
    assert bench.main(["--impl", "reference", "--gpus", "2"]) == 0
