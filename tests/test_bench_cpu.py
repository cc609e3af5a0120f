"""bench.py's host-side logic on CPU: the reference arm (the fp64 oracle on a bounded sample) prints
one well-formed JSON line, and the multi-rank plumbing (process group, barrier, max over ranks, the
reference arm's rank-0-only output) works with two gloo ranks."""

import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    return env


def test_reference_arm_prints_one_json_line():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
         "tiny_gqa", "--steps", "2", "--warmup", "1", "--cpu-sample-tokens", "4096"],
        capture_output=True, text=True, timeout=300, env=_env(0, 1, _free_port()))
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "us/step" and d["value"] > 0
    assert d["higher_is_better"] is False and d["steps"] == 2 and d["warmup"] == 1
    assert d["config"]["workload"] == "tiny_gqa"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


_RANK_SCRIPT = r"""
import sys, json
sys.argv = ["bench.py", "--gpus", "2"]
import bench
args = bench.parse()
rank, world, local = bench.dist_init(args)
bench.barrier(world)
m = bench.max_over_ranks(1.5 + 10.0 * rank, world)
bench.barrier(world)
print(json.dumps({"rank": rank, "world": world, "max": m}), flush=True)
import torch.distributed as dist
dist.destroy_process_group()
"""


def _run_ranks(cmd_for_rank, world=2, timeout=240):
    port = _free_port()
    procs = [subprocess.Popen(cmd_for_rank(r), stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                              text=True, env=_env(r, world, port), cwd=ROOT)
             for r in range(world)]
    outs = []
    try:
        for p in procs:
            o, e = p.communicate(timeout=timeout)
            outs.append((p.returncode, o, e))
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
    return outs


def test_two_gloo_ranks_agree_on_the_max_step_time():
    outs = _run_ranks(lambda r: [sys.executable, "-c", _RANK_SCRIPT])
    for rc, o, e in outs:
        assert rc == 0, e
    got = [json.loads(o.strip().splitlines()[-1]) for _, o, _ in outs]
    assert sorted(g["rank"] for g in got) == [0, 1]
    assert all(g["world"] == 2 and g["max"] == 11.5 for g in got)


def test_reference_arm_under_two_ranks_prints_on_rank_zero_only():
    outs = _run_ranks(lambda r: [sys.executable, os.path.join(ROOT, "bench.py"), "--impl",
                                 "reference", "--gpus", "2", "--workload", "tiny_gqa",
                                 "--steps", "1", "--warmup", "0", "--cpu-sample-tokens", "4096"])
    for rc, o, e in outs:
        assert rc == 0, e
    printed = [[l for l in o.splitlines() if l.strip()] for _, o, _ in outs]
    assert len(printed[0]) == 1 and json.loads(printed[0][0])["n_gpus"] == 2
    assert printed[1] == []
