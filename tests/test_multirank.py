"""Multi-rank host logic of the benchmark, on CPU with gloo process groups.

Token rows are independent, so an N-GPU run gives every rank its own block of
T tokens with the same factors, channel scales and alpha, runs no collective on
the data path, and reports the slowest rank's time with the tokens of all
ranks.  These tests run that logic with world_size 2 on the CPU: the shards,
the max-over-ranks reduction, the whole-job value, per-shard oracle results,
and the reference arm's rank handling.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, init_file, out_dir):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    from kronecker_factored_transforms_b200.workloads import make_workload

    dist.init_process_group("gloo", init_method="file://" + init_file, rank=rank,
                            world_size=world)
    try:
        w = make_workload("hidden8192", rows=8, shard=rank)
        # per-rank "elapsed times" that differ: every rank must see the max
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"), world)
        value = bench.whole_job_tokens_per_s(world, w.T, 4, ms)
        oracle.build()
        r = oracle.transform_quant(w.x, w.P1, w.P2, w.cinv, w.alpha, w.n1, w.n2, nthreads=2)
        q, s = r["packed"], r["scale32"]
        dist.barrier()
        np.savez(os.path.join(out_dir, "rank%d.npz" % rank), x=w.x, P1=w.P1, P2=w.P2,
                 cinv=w.cinv, alpha=np.float32(w.alpha), T=w.T, ms=ms, value=value,
                 q=q, s=s)
    finally:
        dist.destroy_process_group()


def _run_world(world, tmp):
    import torch.multiprocessing as mp
    init_file = os.path.join(tmp, "init")
    mp.start_processes(_worker, args=(world, init_file, tmp), nprocs=world, join=True,
                       start_method="spawn")
    return [dict(np.load(os.path.join(tmp, "rank%d.npz" % r))) for r in range(world)]


@pytest.fixture(scope="module")
def two_ranks(tmp_path_factory):
    return _run_world(2, str(tmp_path_factory.mktemp("gloo2")))


def test_shards_share_factors_not_rows(two_ranks):
    r0, r1 = two_ranks
    for k in ("P1", "P2", "cinv", "alpha"):
        assert np.array_equal(r0[k], r1[k]), k
    assert r0["x"].shape == r1["x"].shape
    assert not np.array_equal(r0["x"], r1["x"])


def test_shard_is_deterministic(two_ranks):
    from kronecker_factored_transforms_b200.workloads import make_workload
    for r, d in enumerate(two_ranks):
        again = make_workload("hidden8192", rows=8, shard=r)
        assert np.array_equal(again.x, d["x"])


def test_shard0_matches_single_gpu_rows(two_ranks):
    """Rank 0 of a multi-GPU run processes the same rows as a 1-GPU run."""
    from kronecker_factored_transforms_b200.workloads import make_workload
    assert np.array_equal(make_workload("hidden8192", rows=8).x, two_ranks[0]["x"])


def test_time_is_max_over_ranks(two_ranks):
    for d in two_ranks:
        assert float(d["ms"]) == 15.0


def test_value_counts_all_ranks(two_ranks):
    for d in two_ranks:
        T = int(d["T"])
        assert float(d["value"]) == pytest.approx(2 * T * 4 / 15e-3)


def test_each_rank_quantises_its_own_rows(two_ranks, oracle_mod):
    """No rank needs another rank's data: the oracle on each shard alone gives
    that rank's result, and the two shards' results differ."""
    for d in two_ranks:
        r = oracle_mod.transform_quant(d["x"], d["P1"], d["P2"], d["cinv"], float(d["alpha"]),
                                       64, 128)
        q, s = r["packed"], r["scale32"]
        assert np.array_equal(q, d["q"])
        assert np.array_equal(s, d["s"])
    assert not np.array_equal(two_ranks[0]["q"], two_ranks[1]["q"])


def test_single_rank_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, 1) == 3.5
    assert bench.whole_job_tokens_per_s(1, 8192, 10, 1000.0) == pytest.approx(81920.0)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_line():
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1", "--ref-seconds", "1.5"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
