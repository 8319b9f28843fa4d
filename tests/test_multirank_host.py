"""Multi-rank host path on CPU (gloo, world size 2): the max-over-ranks
timing, the replica aggregation, the reference arm under torchrun, and a
rank that leaves -- all without a GPU."""
import json
import os
import socket
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORKER = os.path.join(ROOT, "tests", "multirank_worker.py")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port, **extra):
    env = dict(os.environ)
    env.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
               LOCAL_RANK=str(rank), WORLD_SIZE=str(world), CUDA_VISIBLE_DEVICES="")
    env.update({k: str(v) for k, v in extra.items()})
    return env


def _run_ranks(mode, world=2, timeout=120, **extra):
    port = _free_port()
    procs = [subprocess.Popen([sys.executable, WORKER, mode], env=_env(r, world, port, **extra),
                              stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
             for r in range(world)]
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=timeout)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        outs.append((p.returncode, o, e))
    return outs


def _json_line(text):
    lines = [ln for ln in text.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, text
    return json.loads(lines[0])


def test_max_over_ranks_and_replica_value():
    outs = _run_ranks("max")
    seen = []
    for rc, o, e in outs:
        assert rc == 0, e
        seen.append(_json_line(o))
    assert {d["rank"] for d in seen} == {0, 1}
    for d in seen:
        assert d["backend"] == "gloo" and d["world"] == 2
        assert d["max"] == 2.5                      # the slower rank's time, on every rank
        # 2 replicas x 4 MB per 2.5 ms step = 3.2 GB/s for the whole job
        assert abs(d["value"] - 3.2) < 1e-12


def test_departed_rank_ends_the_collective_with_an_error():
    t0 = time.time()
    outs = _run_ranks("dead_peer", PG_TIMEOUT_S=5, timeout=150)
    by_rank = {}
    for rc, o, e in outs:
        assert rc == 0, e
        d = _json_line(o)
        by_rank[d["rank"]] = d
    assert by_rank[0]["error"] is not None          # an error, not a hang
    assert time.time() - t0 < 150


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    port = _free_port()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "2", "--warmup", "3", "--workload", "parity_512x512_t4"]
    r = subprocess.run(cmd, env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    d = _json_line(r.stdout)
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["value"] > 0 and d["unit"] == "GB/s"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
