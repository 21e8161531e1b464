"""Host side of the N > 1 bench path, on CPU with gloo ranks: the max over
ranks that every multi-GPU timing goes through, the per-rank inputs of the
weak-scaling run, and the reference arm under torchrun (rank 0 alone runs
the oracle and prints the one JSON line, the other rank exits without
work)."""
import json
import os
import socket
import subprocess
import sys
import tempfile

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import bench
    v = bench.max_over_ranks(1.5 * (rank + 1), True, torch.device("cpu"))
    bench.barrier(True)
    with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
        f.write(repr(v))
    torch.distributed.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    port = _free_port()
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank_main, args=(2, port, d), nprocs=2, start_method="spawn")
        vals = [float(open(os.path.join(d, f"r{r}.txt")).read()) for r in range(2)]
    assert vals == [3.0, 3.0]


def test_per_rank_inputs_differ_but_share_weights():
    import bench
    a = bench.make_inputs(4, "cpu", seed_offset=0)
    b = bench.make_inputs(4, "cpu", seed_offset=bench.RANK_SEED_STRIDE)
    for name in bench.PROJ:
        assert torch.equal(a[name][3], b[name][3])          # W
        assert not torch.equal(a[name][2], b[name][2])      # X


def test_step_refuses_activations_shorter_than_m():
    """The library reads M rows of X through a raw pointer, so the bench step
    checks the host tensor before anything is allocated or launched."""
    import pytest
    import bench
    data = bench.make_inputs(16, "cpu")
    with pytest.raises(ValueError, match="needs at least 32"):
        bench.Step(None, data, 32, "cpu")


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-rows", "1"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(l) for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    d = lines[0]
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
