"""Multi-process (gloo, world size 2, CPU) checks of bench.py's N-GPU logic.

bench.py runs one replica of the matrix set per rank (weak scaling, no
collective on the data path); the only collectives are the barrier and the
max over ranks of the timed region.  These run here without a GPU.
"""
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = 100.0 + 25.0 * rank          # the slower rank decides
        ms = bench.reduce_max(ms_local, "cpu")
        value = bench.aggregate_value(224, world, ms)
        dist.barrier()
        out[rank] = (ms, value, bench.dist_env())
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        ms, value, env = res[rank]
        assert ms == 125.0                       # max over ranks on every rank
        assert abs(value - 2 * 224 / 0.125) < 1e-9
        assert env == (rank, world, rank)


def test_reduce_max_without_process_group_is_identity():
    assert bench.reduce_max(3.5, "cpu") == 3.5
    assert bench.aggregate_value(224, 1, 500.0) == 448.0


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"]))
    assert capsys.readouterr().out == ""


def test_e2e_groups_cover_every_matrix_once():
    import workloads
    for w in workloads.WORKLOADS:
        groups = bench.e2e_groups(w)
        flat = sorted(i for g in groups for i in g)
        assert flat == list(range(w.count))
        for g in groups:
            shapes = {(min(*w.shapes[i]), max(*w.shapes[i])) for i in g}
            assert len(shapes) == 1 and len(g) <= 16
