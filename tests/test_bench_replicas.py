"""The bench's multi-process plumbing on CPU (gloo, world size 2): replicas, barrier, max over ranks.

The decode path shards by independent replicas (one per GPU) with no exchange
between them; the only collectives are the barrier around the timed region and
the max of the per-rank step times.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


WORKER = r"""
import os, sys, datetime
sys.path.insert(0, sys.argv[1])
import torch.distributed as dist
import bench
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
rank = dist.get_rank()
bench.dist_barrier(2)
m = bench.dist_max(1.5 + rank, 2)
assert m == 2.5, m
dist.destroy_process_group()
print("ok", rank)
"""


def test_max_over_ranks_and_barrier_with_gloo(tmp_path):
    script = tmp_path / "worker.py"
    script.write_text(WORKER)
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script), ROOT], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = [p.communicate(timeout=240)[0] for p in procs]
    for rank, (p, out) in enumerate(zip(procs, outs)):
        assert p.returncode == 0, out
        assert f"ok {rank}" in out


def test_reference_arm_under_torchrun_prints_one_line(tmp_path):
    """`bench.py --impl reference` under torchrun: rank 0 times the oracle, rank 1 exits cleanly."""
    port = _free_port()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3", "--config", "1",
           "--reference-budget", "1"]
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=600, cwd=str(tmp_path))
    assert r.returncode == 0, r.stdout + r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    import json
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_maps_no_product_library_and_shares_the_config():
    """The oracle's arm loads the oracle's library only, and its `config` is the GPU line's."""
    code = ("import sys, json, io, contextlib; sys.path.insert(0, %r); import bench\n"
            "buf = io.StringIO()\n"
            "with contextlib.redirect_stdout(buf):\n"
            "    bench.main(['--impl', 'reference', '--steps', '1', '--warmup', '3', '--config', '1',"
            " '--reference-budget', '0.5'])\n"
            "maps = open('/proc/self/maps').read()\n"
            "assert 'libpagedkv' not in maps, 'product library mapped'\n"
            "line = json.loads([l for l in buf.getvalue().splitlines() if l.startswith('{')][0])\n"
            "from paged_kv_cache_470_b200 import workloads\n"
            "cfg = workloads.WORKLOADS[1]\n"
            "assert line['config'] == bench.config_record(cfg, workloads.draw_layout(cfg), 1), line['config']\n"
            "print('ok')") % ROOT
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
