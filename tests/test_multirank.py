"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

Pairs are independent problems, so a run on N GPUs is N replicas that each match
their own slice of the pair stream with no collective on the data path; the only
cross-rank step is the max of the per-rank step times.  These tests check, with
world_size 2 on the gloo backend:
  * the shards of the ranks are disjoint and cover the stream in order,
  * a pair's synthetic inputs do not depend on which rank generates them,
  * the float64 oracle run on each rank's shard, gathered, equals one run over
    the whole stream (the sharding is exact, so no data exchange is needed),
  * the reported step time is the slowest rank's and the throughput counts the
    pairs of every rank.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORLD = 2
PAIRS_PER_RANK = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _small_workload():
    from learned_sparse_feature_b200 import synth
    w = synth.WORKLOADS["pair64_fp32"]
    return w


def _rank_main(rank, port, out_q):
    import torch.distributed as dist

    import bench
    from learned_sparse_feature_b200 import synth
    from oracle import superglue_oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        w = _small_workload()
        first = bench.shard_pairs(PAIRS_PER_RANK, rank)
        batch = synth.make_batch(w, first, PAIRS_PER_RANK)
        weights = synth.make_weights(0)
        # a shortened network keeps the float64 oracle quick; the sharding
        # argument does not depend on the depth
        res = O.superglue_batch(batch, weights, n_stages=2, iters=20)
        local = {
            "first": first,
            "kpts0": batch["kpts0"],
            "matches0": np.stack([r["matches0"] for r in res]),
            "mscores0": np.stack([r["mscores0"] for r in res]),
        }
        gathered = [None] * WORLD
        dist.all_gather_object(gathered, local)
        # per-rank "step times": rank r took 10 + 5 r ms in total
        t_max = bench.reduce_max(10.0 + 5.0 * rank, dist)
        rate = bench.whole_job_rate(PAIRS_PER_RANK, dist.get_world_size(), 4, t_max)
        dist.barrier()
        if rank == 0:
            out_q.put({"gathered": gathered, "t_max": t_max, "rate": rate})
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_rank_run():
    import multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    try:
        out = q.get(timeout=300)
    finally:
        for p in procs:
            p.join(timeout=120)
    for p in procs:
        assert p.exitcode == 0, f"rank process exited with {p.exitcode}"
    return out


def test_shards_disjoint_and_ordered():
    import bench
    firsts = [bench.shard_pairs(PAIRS_PER_RANK, r) for r in range(WORLD)]
    covered = [i for f in firsts for i in range(f, f + PAIRS_PER_RANK)]
    assert covered == list(range(WORLD * PAIRS_PER_RANK))


def test_rank_inputs_match_unsharded_stream(two_rank_run):
    from learned_sparse_feature_b200 import synth
    w = _small_workload()
    full = synth.make_batch(w, 0, WORLD * PAIRS_PER_RANK)
    for r, g in enumerate(two_rank_run["gathered"]):
        assert g["first"] == r * PAIRS_PER_RANK
        np.testing.assert_array_equal(g["kpts0"], full["kpts0"][g["first"]:g["first"] + PAIRS_PER_RANK])


def test_sharded_oracle_equals_unsharded(two_rank_run):
    from learned_sparse_feature_b200 import synth
    from oracle import superglue_oracle as O
    w = _small_workload()
    full = synth.make_batch(w, 0, WORLD * PAIRS_PER_RANK)
    res = O.superglue_batch(full, synth.make_weights(0), n_stages=2, iters=20)
    m0 = np.concatenate([g["matches0"] for g in two_rank_run["gathered"]])
    s0 = np.concatenate([g["mscores0"] for g in two_rank_run["gathered"]])
    np.testing.assert_array_equal(m0, np.stack([r["matches0"] for r in res]))
    np.testing.assert_array_equal(s0, np.stack([r["mscores0"] for r in res]))


def test_step_time_is_slowest_rank_and_rate_counts_all_ranks(two_rank_run):
    assert two_rank_run["t_max"] == 15.0
    # 2 ranks x 2 pairs x 4 steps in 15 ms
    assert two_rank_run["rate"] == pytest.approx(16 / 0.015)
