"""The multi-process path of bench.py, on CPU with the gloo backend.

The work path has no exchange step: every rank runs an independent replica and
the timing is the maximum over ranks.  These tests run two ranks on the host:
the max-over-ranks reduction and barrier used by the bench, and the reference
arm under torchrun (rank 0 prints one JSON line, rank 1 exits cleanly).
"""
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
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        got = bench.max_over_ranks(float(rank + 1) * 1.5, world)
        bench.barrier(world)
        with open(f"{out_path}.{rank}", "w") as f:
            f.write(repr(got))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_gloo(tmp_path):
    port = _free_port()
    out = str(tmp_path / "res")
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(2):
        assert float(open(f"{out}.{r}").read()) == 3.0


def test_reference_arm_under_torchrun(tmp_path):
    env = dict(os.environ)
    env.pop("CUDA_VISIBLE_DEVICES", None)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "3", "--workload", "grid16_f32"]
    r = subprocess.run(cmd, cwd=str(tmp_path), env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_workload_byte_and_flop_accounting():
    """The bench's algorithmic figures: q, k, v read and out written once (e4m3
    inputs at one byte, their bf16 output at two), and 4·B·H·d flops per
    (query, key) pair that the method computes."""
    sys.path.insert(0, ROOT)
    import bench
    from basa_synth import WORKLOADS
    w16, w8 = WORKLOADS["flux2048"], WORKLOADS["flux2048_e4m3"]
    f16, b16, N, m, P, theo = bench.workload_numbers(w16, (0, 8, 8))
    f8, b8, *_ = bench.workload_numbers(w8, (0, 8, 8))
    assert b16 == 4 * 24 * 16384 * 128 * 2
    assert b8 == 24 * 16384 * 128 * (3 * 1 + 2)
    assert f16 == f8 == 4.0 * 24 * 128 * 16384 * 256
    assert theo == 16384 / 256
    fj, bj, N, m, P, theo = bench.workload_numbers(WORKLOADS["flux1024_text512"], (0, 8, 8))
    L = 512
    assert fj == 4.0 * 24 * 128 * (4096 * (256 + L) + L * (4096 + L))
    assert bj == 4 * 24 * (4096 + L) * 128 * 2


def test_reference_arm_backward_and_joint(tmp_path):
    """The reference arm times the oracle's backward under --backward, and the
    joint forward (image and text queries) for a joint workload."""
    def run(*extra):
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                            "--steps", "1", "--warmup", "1", *extra],
                           capture_output=True, text=True, timeout=600, cwd=ROOT)
        assert r.returncode == 0, r.stderr[-2000:]
        return json.loads(r.stdout.strip().splitlines()[-1])
    j = run("--backward", "--workload", "grid16_f32")
    assert j["impl"] == "reference" and j["metric"].startswith("window-attn backward")
    assert j["value"] > 0 and j["cpu_baseline"]["cores"] == 1
    j = run("--workload", "flux1024_text512")
    assert "text queries" in j["cpu_baseline"]["sample"] and j["value"] > 0
