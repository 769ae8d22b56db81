"""The multi-rank path on host cores (gloo, world size 2): one process per rank, the timing
helpers of the benchmark (barrier, maximum over ranks), the per-rank workloads of weak
scaling, and the reference arm run under torchrun (rank 0 alone works and prints one line;
the other rank exits 0 without work)."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup()
    assert (w, r) == (ws, rank) and dist.get_backend() == "gloo"
    bench.dist_barrier(w)
    got = bench.dist_max(1.5 * (rank + 1), w)
    sp = bench.rank_spec("tiny", rank)
    from long_context_kv_srht_b200 import workload
    first_key = workload.generate(workload.spec(sp.name, n=64, seed=sp.seed)).keys[0, 0, 0]
    np.save(os.path.join(out_dir, f"r{rank}.npy"), np.concatenate([[got], first_key]))
    bench.dist_barrier(w)
    dist.destroy_process_group()


def test_timing_helpers_and_rank_workloads(tmp_path):
    ws = 2
    mp.spawn(_rank_main, args=(ws, _free_port(), str(tmp_path)), nprocs=ws, join=True)
    r0, r1 = (np.load(tmp_path / f"r{r}.npy") for r in range(ws))
    assert r0[0] == r1[0] == 3.0                       # max over ranks seen by every rank
    assert not np.array_equal(r0[1:], r1[1:])          # every rank has its own sequences


def test_reference_arm_two_ranks():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node",
           "2", "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["config"]["workload"] == "tiny" and line["steps"] == 2 and line["warmup"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert {"value", "unit", "sample"} <= set(cb)
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
