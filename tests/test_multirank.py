"""The multi-rank plumbing of bench.py on the CPU: two gloo ranks (world size 2) initialise
the process group, agree on the maximum time and sum the ranks' tokens; each rank routes
its own batch; the reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    from workloads import BEAM, activations
    w, r, _ = bench.init_dist()
    assert (w, r) == (world, rank)
    elapsed = 100.0 + 10.0 * rank               # a different time on every rank
    bench.barrier(w)
    m = bench.max_over_ranks(elapsed, w)
    x = activations(4, BEAM, seed=rank)          # each rank's own batch
    torch.distributed.destroy_process_group()
    out[rank] = (m, bench.tokens_per_second(w, 16, 10, m), float(x.float().sum()))


def test_two_gloo_ranks_reduce_time_and_sum_tokens():
    world = 2
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 110.0                       # max over ranks
    assert res[0][1] == res[1][1] == pytest.approx(2 * 16 * 10 / 0.110)
    assert res[0][2] != res[1][2]                                # different batches per rank


def test_reference_arm_rank0_only_and_json_line():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny", "--steps", "2", "--warmup", "1"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert p.returncode == 0 and p.stdout.strip() == ""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny", "--steps", "2", "--warmup", "1"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert p.returncode == 0, p.stderr
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
