"""bench.py's multi-rank host logic (one process per GPU on a real run) with
world_size 2 over gloo on CPU: rank-specific inputs, max-over-ranks timing,
barrier, the reference arm running on rank 0 only, and the launcher that
``--gpus N`` starts when no WORLD_SIZE is set."""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, wsz, lr = bench.dist_env()
        assert (r, wsz, lr) == (rank, world, rank)
        t = [1.0 + rank, 10.0 - rank]
        m = bench.reduce_max(t, wsz)
        bench.barrier(wsz)
        w = bench.rank_workload(bench.HEADLINE, rank)
        q.put((rank, m, w.seed, None))
    finally:
        dist.destroy_process_group()


def test_two_rank_host_logic():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, s0, _), (r1, m1, s1, _) = out
    assert m0 == m1 == [2.0, 10.0]          # element-wise max over ranks
    assert s0 != s1                           # each rank runs its own batch


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    class A:
        steps, warmup = 1, 0
    assert bench.run_reference(A, 1, 2) is None
    line = bench.run_reference(A, 0, 1)
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_gpus_flag_launches_that_many_ranks(tmp_path, capfd, monkeypatch):
    """`bench.py --gpus 2` without a launcher starts two rank processes itself;
    rank 0 prints the one JSON line with n_gpus 2."""
    sys.path.insert(0, ROOT)
    import bench
    for v in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(v, raising=False)
    log = tmp_path / "ranks.txt"
    rc = bench.main(["--gpus", "2", "--impl", "reference", "--steps", "1", "--warmup", "3",
                     "--ranks-log", str(log)])
    assert rc == 0
    lines = sorted(log.read_text().split("\n")[:-1])
    assert [ln.split()[:2] for ln in lines] == [["0", "2"], ["1", "2"]]
    assert len({ln.split()[2] for ln in lines}) == 2          # two processes
    out = [ln for ln in capfd.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(out) == 1                                       # rank 0 alone prints
    rec = json.loads(out[0])
    assert rec["n_gpus"] == 2 and rec["impl"] == "reference"


def test_gpus_flag_disagreeing_with_launcher_fails(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    assert bench.main(["--gpus", "2", "--impl", "reference", "--steps", "1", "--warmup", "3"]) == 2
