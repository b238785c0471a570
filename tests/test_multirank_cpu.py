"""The multi-rank path on CPU: two gloo ranks (world size 2).

Each rank owns its own batch of requests (weak scaling) and steps it with no
exchange on the data path; only the timing crosses ranks (a barrier and the
maximum of the ranks' times).  The ranks here run the oracle step on their
pages (no GPU in this test) and must get exactly what one process gets for
the same rank's batch, so sharding changes nothing.  The benchmark's
reference arm prints from rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import torch.multiprocessing as mp

from linear_attention_recurrent_delta_b200 import ranks as R
from linear_attention_recurrent_delta_b200 import workloads as W

from parity_util import oracle_quantize, oracle_step

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2


def _workload():
    return W.WORKLOADS[2].resized(batch=2, heads=3, steps=1)


def _rank_result(rank):
    """A rank's step on its own pages (oracle): returns (pages after, o)."""
    wr = R.rank_workload(_workload(), rank)
    S = W.initial_state(wr).numpy()
    fmt, perm, pages = oracle_quantize(wr, S)
    x = W.step_inputs(wr, 0)
    return oracle_step(fmt, wr, wr.batch, wr.heads, pages, perm, x, W.sr_seed(wr), 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    world, r, _ = R.init("gloo", timeout_s=60)
    assert (world, r) == (WORLD, rank)
    pages, o = _rank_result(rank)
    R.barrier(world)
    t_ms = 10.0 * (1 + rank)                       # stand-in for this rank's device time
    t_max = R.max_over_ranks(t_ms, world)
    rate = R.aggregate_rate(_workload().pages, world, 5, t_max)
    np.savez(os.path.join(outdir, "rank%d.npz" % rank), pages=pages, o=o, t_max=t_max, rate=rate,
             seed=R.rank_workload(_workload(), rank).seed)
    R.finish(world)


def test_two_gloo_ranks_step_their_own_pages(tmp_path):
    mp.start_processes(_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD, start_method="spawn")
    res = [np.load(os.path.join(tmp_path, "rank%d.npz" % r)) for r in range(WORLD)]
    for r in res:
        assert float(r["t_max"]) == 20.0                       # the slower rank's time
        assert float(r["rate"]) == _workload().pages * WORLD * 5 / 0.020
    assert int(res[0]["seed"]) != int(res[1]["seed"])          # each rank its own requests
    assert not np.array_equal(res[0]["o"], res[1]["o"])
    for rank in range(WORLD):                                  # sharding changes nothing
        pages, o = _rank_result(rank)
        assert np.array_equal(res[rank]["pages"], pages)
        assert np.array_equal(res[rank]["o"], o)


def test_rank_helpers_alone():
    assert R.max_over_ranks(3.5, 1) == 3.5
    assert R.aggregate_rate(100, 4, 10, 2.0) == 100 * 4 * 10 / 0.002
    w = _workload()
    assert R.rank_workload(w, 0) == w
    assert R.rank_workload(w, 3).seed == w.seed + 3 * R.RANK_SEED_STRIDE


def _bench_reference(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "0",
                           "--steps", "2", "--warmup", "1", "--ref-seconds", "1"],
                          env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_on_rank_zero_only():
    other = _bench_reference(1)
    assert other.returncode == 0, other.stderr
    assert other.stdout.strip() == ""
    first = _bench_reference(0)
    assert first.returncode == 0, first.stderr
    line = json.loads(first.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == WORLD
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
