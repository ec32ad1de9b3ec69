"""The host logic of bench.py's multi-GPU run (one process per GPU, replicas
with no collective on the data path) with two gloo ranks on the CPU: the
max-over-ranks step time, the whole-job aggregate and the reference arm's
rank-0-only rule."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out_dir):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(ws), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, local = bench.dist_env()
        ms = bench.max_over_ranks(1.0 + 2.5 * rank, w, "cpu")         # rank 1 is the slow one
        ms2 = bench.max_over_ranks(7.0 - rank, w, "cpu")
        gbs = bench.whole_job_gbs(w, 641728512, ms)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"ws": w, "rank": r, "local": local, "ms": ms, "ms2": ms2, "gbs": gbs}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_max_and_the_aggregate(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    for r, d in enumerate(res):
        assert (d["ws"], d["rank"], d["local"]) == (2, r, r)
        assert d["ms"] == 3.5 and d["ms2"] == 7.0                     # every rank gets the slowest time
        assert d["gbs"] == pytest.approx(2 * 641728512 / 3.5e-3 / 1e9)  # both ranks' bytes over it


def test_reference_arm_runs_on_rank_0_only():
    """Under torchrun the reference arm prints on rank 0; another rank exits
    0 at once, without output and without touching the oracle."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0
    assert p.stdout.strip() == ""
