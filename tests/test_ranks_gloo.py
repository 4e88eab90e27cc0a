"""The replicas' host plumbing with two ranks on CPU (gloo over 127.0.0.1):
bench.Ranks' barrier, maximum over ranks and whole-job aggregate, and the
reference arm's rule that only rank 0 does work and prints."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys
sys.path.insert(0, sys.argv[1])
import torch
import bench
r = bench.Ranks("gloo", torch.device("cpu"))
r.barrier()
m = r.max(1.5 + r.rank)                        # rank 1 is the slower one
agg = r.aggregate(10.0, 2.0 + 3.0 * r.rank)    # 10 units per rank; 2 ms and 5 ms
r.barrier()
r.close()
print(json.dumps(dict(rank=r.rank, ws=r.ws, max=m, agg=agg)))
"""


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_barrier_max_and_aggregate():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", CHILD, ROOT], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    try:
        for p in procs:
            outs.append(p.communicate(timeout=180))
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
    for p, (_, err) in zip(procs, outs):
        assert p.returncode == 0, err[-2000:]
    res = sorted((json.loads(o.strip().splitlines()[-1]) for o, _ in outs), key=lambda d: d["rank"])
    assert [d["rank"] for d in res] == [0, 1]
    for d in res:
        assert d["ws"] == 2
        assert d["max"] == 2.5
        # 2 ranks x 10 units over the slower rank's 5 ms
        assert abs(d["agg"] - 2 * 10.0 / 5e-3) < 1e-9


def test_single_process_needs_no_process_group():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    env = {k: os.environ.pop(k) for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK") if k in os.environ}
    try:
        r = bench.Ranks("gloo", torch.device("cpu"))
        assert (r.ws, r.rank) == (1, 0)
        r.barrier()
        assert r.max(3.25) == 3.25
        assert r.aggregate(4.0, 2.0) == 4.0 / 2e-3
        r.close()
    finally:
        os.environ.update(env)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=180)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""
