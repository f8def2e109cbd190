"""Multi-rank plumbing of the replicas path, as world_size-2 gloo process groups on the CPU.

The decode step has no exchange between GPUs. N GPUs run N replicas, timed as the maximum
over ranks, with throughput summed over ranks. These tests check that host logic
with real gloo ranks:
* the max reduction;
* the whole-job rate;
* the barrier;
* a rank that never arrives ends the others' collective with an error instead of a hang;
* bench.py's reference arm under torchrun: only rank 0 prints, and every rank exits 0.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    from rotated_bit_matmul_b200 import replicas
    rk = replicas.from_env()
    replicas.init(rk, "gloo", timeout_s=60)
    replicas.barrier(rk)
    ms_local = 10.0 + 5.0 * rank  # rank 1 is the slow one
    ms = replicas.max_over_ranks(rk, ms_local)
    rate = replicas.whole_job_rate(rk, 50, ms)
    replicas.finish(rk)
    q.put((rank, rk.world, ms, rate))


def _silent_rank_main(rank, world, port, q):
    """Rank 1 joins the group and then leaves without joining the collective."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    from rotated_bit_matmul_b200 import replicas
    import torch.distributed as dist
    rk = replicas.from_env()
    replicas.init(rk, "gloo", timeout_s=5)
    if rank == 0:
        try:
            replicas.max_over_ranks(rk, 1.0)
            q.put((rank, "returned"))
        except Exception as e:  # the short process-group timeout ends the collective
            q.put((rank, "error:" + type(e).__name__))
    else:
        q.put((rank, "left"))
    try:
        dist.destroy_process_group()
    except Exception:
        pass


def _spawn(fn, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    return sorted(out), [p.exitcode for p in procs]


def test_single_rank_is_identity():
    from rotated_bit_matmul_b200 import replicas
    rk = replicas.Ranks(0, 1, 0)
    assert replicas.max_over_ranks(rk, 3.5) == 3.5
    assert replicas.whole_job_rate(rk, 100, 1000.0) == pytest.approx(100.0)
    with pytest.raises(ValueError):
        replicas.whole_job_rate(rk, 1, 0.0)


def test_two_ranks_max_and_rate():
    out, codes = _spawn(_rank_main, 2)
    assert codes == [0, 0]
    for rank, world, ms, rate in out:
        assert world == 2
        assert ms == 15.0  # the slow rank's time on every rank
        assert rate == pytest.approx(2 * 50 / 0.015)  # units of both ranks over the max time


def test_missing_rank_errors_instead_of_hanging():
    out, codes = _spawn(_silent_rank_main, 2)
    d = dict(out)
    assert d[1] == "left"
    assert d[0].startswith("error:")


def test_bench_reference_arm_two_ranks():
    """bench.py --impl reference under torchrun with 2 ranks: rank 0 prints one JSON line
    carrying impl=reference; rank 1 exits 0 without output."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(["timeout", "-k", "30", "600", *cmd], cwd=ROOT, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["config"]["parallelism"] == "replicas2"
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
