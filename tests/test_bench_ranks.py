"""bench.py's multi-rank plumbing on the host, over gloo with two ranks: the max-over-ranks
reduction that the timing uses, and the reference arm under torchrun (rank 0 alone runs the
oracle and prints one JSON line; the other rank exits 0 without work). No GPU is used."""
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


def _max_worker(rank, port, out_dir):
    import datetime
    import torch
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=2,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        v = bench.max_over_ranks(1.5 * (rank + 1), 2)   # rank 0: 1.5, rank 1: 3.0
        bench.barrier(2)
        with open(os.path.join(out_dir, f"r{rank}"), "w") as f:
            f.write(repr(v))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks(tmp_path):
    mp.start_processes(_max_worker, args=(_free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for r in range(2):
        assert float((tmp_path / f"r{r}").read_text()) == 3.0


@pytest.mark.timeout(300)
def test_reference_arm_two_ranks_prints_one_line(orc):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "llama2_7b_qproj_b1"]
    env = dict(os.environ, OMP_NUM_THREADS="1", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=280)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["value"] > 0 and rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["d2h_bytes_per_step"] == 0
