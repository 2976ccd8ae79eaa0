"""Host-side logic of bench.py on CPU: the max-over-ranks reduction and the
whole-job value across world_size-2 gloo ranks, and the reference arm's JSON."""

import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    times = [1.0 + rank, 0.1 * (rank + 1)]
    mx = bench.reduce_max(times, world)
    val = bench.whole_job_value(100.0, world, mx[0])
    dist.destroy_process_group()
    q.put((rank, mx, val))


def test_max_over_ranks_and_whole_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, val in res:
        assert mx == [2.0, 0.2]                 # max over ranks, every rank sees it
        assert val == pytest.approx(100.0 * 2 / 2.0)


def test_reference_arm_prints_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "cpu_baseline", "e2e", "config"):
        assert key in line
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


@pytest.mark.parametrize("d,h,rounds", [(256, 64, 1), (512, 128, 2), (384, 128, 3), (1024, 256, 1)])
def test_sweep_rotation_equals_the_oracle(d, h, rounds):
    # the sweep's own fp64 torch rotation (used for its MSE figures) against the
    # oracle's dense composed rotation, on the oracle's draws of the same seed
    import numpy as np
    import torch
    sys.path.insert(0, ROOT)
    import bench
    from oracle import rpbh
    R = rpbh.draw_rounds(0, d, rounds)
    X = np.random.default_rng(d + rounds).standard_normal((7, d))
    X[3] = 0.0
    X[3, 11] = 2.0                              # a one-hot row
    tables = [(torch.from_numpy(np.asarray(p, dtype=np.int64)), torch.from_numpy(np.asarray(s, dtype=np.float64)))
              for p, s in R]
    got = bench.rotate_rows_f64(torch.from_numpy(X), tables, h).numpy()
    ref = rpbh.rotate_composed(X, R, h)
    assert np.allclose(got, ref, rtol=0, atol=1e-12)


def test_workload_cpu_baseline_runs_the_oracle_chain():
    # the oracle leg of `bench.py --workload`: a bounded sample through the same
    # launches the GPU times, with the weights quantized beforehand
    import bench
    dt, flops = bench.oracle_workload_sample("flux_qkv_w3a3", 4)
    assert dt > 0 and flops == 2.0 * 4 * 9216 * 3072
