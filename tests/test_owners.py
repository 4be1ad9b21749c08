"""Dedicated ownership: the load-balanced assignment and the owner's broadcast.

DMuon FAQ, "Why isn't DMuon just ZeRO-1?": one rank owns a whole matrix, runs
its step and broadcasts the updated parameter to the others; Training Guide,
"Verify Parameter Assignment": the assignment is reported with per-rank loads
and an imbalance.  The oracle's assignment is pinned by a hand-computed case and
by brute force (Graham's bound for longest-processing-time-first against the
optimal makespan of tiny sets); the library's equals it exactly.  Two gloo
ranks on the CPU then check the broadcast: every rank ends with its owners'
results bit for bit and touches only the buffers it owns.
"""
import itertools
import os
import random
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import newton_schulz_grad_b200 as nsg
import workloads
from oracle import muon as om


def test_hand_computed_assignment():
    # Newton-Schulz flops per iteration 3 m^2 n + m^3: (2, 2) 32, (1, 5) 16,
    # (1, 3) 10, (1, 2) 7, (1, 1) 4.  Two ranks, most expensive first, each to
    # the lighter rank (ties to rank 0): 32 -> 0, 16 -> 1, 10 -> 1, 7 -> 1, 4 -> 0
    shapes = [(1, 3), (2, 2), (1, 1), (1, 5), (1, 2)]
    owner_of, loads, imbalance = om.assign_owners(shapes, 2)
    assert owner_of == [1, 0, 0, 1, 1]
    assert loads == [36.0, 33.0]
    assert imbalance == pytest.approx(36.0 / 34.5 - 1.0, rel=1e-15)


@pytest.mark.parametrize("seed", range(40))
def test_assignment_within_grahams_bound_of_the_optimum(seed):
    rng = random.Random(seed)
    world = rng.choice([2, 3])
    shapes = [(rng.randint(1, 9), rng.randint(1, 9)) for _ in range(rng.randint(1, 7))]
    owner_of, loads, _ = om.assign_owners(shapes, world)
    cost = [om.ns_iteration_flops(r, c) for r, c in shapes]
    assert sorted(set(owner_of)) <= list(range(world))
    for r in range(world):
        assert loads[r] == pytest.approx(sum(c for c, o in zip(cost, owner_of) if o == r))
    best = min(max(sum(c for c, o in zip(cost, a) if o == r) for r in range(world))
               for a in itertools.product(range(world), repeat=len(shapes)))
    assert max(loads) <= (4.0 / 3.0 - 1.0 / (3.0 * world)) * best + 1e-9


@pytest.mark.parametrize("seed", range(20))
def test_library_assignment_equals_the_oracle(seed):
    rng = random.Random(1000 + seed)
    world = rng.randint(1, 9)
    shapes = [(rng.choice([32, 1024, 1408, 2048, 4096, 11008]), rng.choice([64, 1024, 2048, 4096, 11008]))
              for _ in range(rng.randint(0, 80))]
    got = nsg.dmuon_assign_owners([(r, c, 1) for r, c in shapes], world)
    want = om.assign_owners(shapes, world)
    assert got[0] == want[0] and got[1] == want[1]
    assert got[2] == pytest.approx(want[2], rel=1e-12, abs=1e-15)


def test_llama_7b_set_balances_exactly_over_8_ranks():
    w = workloads.get("llama_7b_bf16")
    owner_of, loads, imbalance = nsg.dmuon_assign_owners([(r, c, 1) for r, c in w.shapes], 8)
    assert imbalance == 0.0 and len(set(owner_of)) == 8


def test_assignment_argument_errors():
    with pytest.raises(nsg.DmuonError):
        nsg.dmuon_assign_owners([(4, 4, 1)], 0)
    with pytest.raises(nsg.DmuonError):
        nsg.dmuon_assign_owners([(0, 4, 1)], 2)
    assert nsg.dmuon_assign_owners([], 3) == ([], [0.0, 0.0, 0.0], 0.0)


# ------------------------------------------------------------ broadcast (gloo)
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_step(ps, gs, bs):
    # the owner's local step, here on the CPU: the fp64 oracle, stored in fp32
    new_p, new_b, _ = om.muon_step([p.double().numpy() for p in ps], [g.double().numpy() for g in gs],
                                   [b.double().numpy() for b in bs], wd=0.1)
    for p, b, q, c in zip(ps, bs, new_p, new_b):
        p.copy_(torch.from_numpy(q).float())
        b.copy_(torch.from_numpy(c).float())


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from newton_schulz_grad_b200.distributed import owned_step
        shapes = [(24, 40), (40, 24), (16, 16), (8, 64), (24, 40), (32, 8)]
        gen = torch.Generator().manual_seed(5)      # the same replicated start on every rank
        params = [torch.randn(r, c, generator=gen) * 0.02 for r, c in shapes]
        grads = [torch.randn(r, c, generator=gen) for r, c in shapes]
        owner_of = om.assign_owners(shapes, world)[0]
        bufs = [torch.zeros(r, c) if owner_of[i] == rank else None for i, (r, c) in enumerate(shapes)]
        seen = []

        def local(ps, gs, bs):
            seen.extend(p.shape for p in ps)
            _oracle_step(ps, gs, bs)

        got = owned_step(params, grads, bufs, local_step=local)
        out[rank] = ([p.numpy().copy() for p in params], [None if b is None else b.numpy().copy() for b in bufs],
                     got[0], seen)
    finally:
        dist.destroy_process_group()


def test_owner_updates_reach_every_rank_bit_for_bit():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    p0, b0, own0, seen0 = res[0]
    p1, b1, own1, seen1 = res[1]
    assert own0 == own1 and set(own0) == {0, 1}
    for a, b in zip(p0, p1):                        # replicated after the broadcast
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    # each matrix holds what its owner computed
    shapes = [(24, 40), (40, 24), (16, 16), (8, 64), (24, 40), (32, 8)]
    gen = torch.Generator().manual_seed(5)
    params = [torch.randn(r, c, generator=gen) * 0.02 for r, c in shapes]
    grads = [torch.randn(r, c, generator=gen) for r, c in shapes]
    bufs = [torch.zeros(r, c) for r, c in shapes]
    _oracle_step(params, grads, bufs)
    for i, p in enumerate(params):
        assert np.array_equal(p.numpy().view(np.uint32), p0[i].view(np.uint32))
        assert (b0[i] is not None) == (own0[i] == 0) and (b1[i] is not None) == (own0[i] == 1)
    assert len(seen0) + len(seen1) == len(shapes)   # every matrix stepped exactly once


@pytest.mark.gpu
def test_owned_step_on_one_gpu_equals_dmuon_step():
    # no process group: one rank owns everything and nothing is broadcast
    from newton_schulz_grad_b200.distributed import owned_step
    w = workloads.get("small_layer_bf16")
    runs = []
    for use_owners in (True, False):
        ps, gs, bs = workloads.make_all(w, "cuda")
        if use_owners:
            owner_of, loads, imbalance = owned_step(ps, gs, bs, wd=0.1)
            assert set(owner_of) == {0} and imbalance == 0.0
        else:
            nsg.dmuon_step(ps, gs, bs, wd=0.1)
        assert nsg.dmuon_stream_status() == nsg.DMUON_OK
        runs.append([t.cpu().view(torch.int16).numpy() for t in ps + bs])
    for a, b in zip(*runs):
        assert np.array_equal(a, b)
