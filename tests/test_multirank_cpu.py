"""The multi-rank path of bench.py on CPU (world size 2, gloo, 127.0.0.1).

The layer's path does not shard across GPUs here: `bench.py --gpus N` runs N
independent replicas, one per rank, and reports the whole job's work over
the slowest rank's device time. These tests run that host logic (the
max-over-ranks reduction and the whole-job throughput) on two gloo ranks,
and the reference arm under torchrun, where rank 0 alone times the oracle
and prints the line while the other rank exits 0 without work."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # ranks with different step times: every rank must see the slowest
        ms = 1.0 + 0.5 * rank
        slowest = bench.max_over_ranks(ms, dist, "cpu")
        value = bench.whole_job_tflops(2.0e12, world, slowest)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "value": value,
                       "alone": bench.max_over_ranks(ms, None, "cpu")}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, g in enumerate(got):
        assert g["slowest"] == 1.5          # rank 1's 1.5 ms, seen by both ranks
        assert g["alone"] == 1.0 + 0.5 * r  # no process group: the rank's own time
        # 2 ranks x 2 TFLOP each over 1.5 ms
        assert g["value"] == pytest.approx(2 * 2.0e12 / 1.5e-3 / 1e12)


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    r = subprocess.run(
        [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
         "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
         "reference", "--gpus", "2", "--workload", "mlp_32x1024_f4096_n2", "--steps", "1",
         "--warmup", "3"],
        cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
