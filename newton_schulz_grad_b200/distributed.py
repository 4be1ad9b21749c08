"""Dedicated ownership across ranks: each matrix stepped by one owner, then broadcast.

DMuon FAQ, "Why isn't DMuon just ZeRO-1?": one rank owns a whole matrix and runs
its Muon step (Newton-Schulz needs the complete matrix); the other ranks receive
the updated parameter by broadcast, which can hide inside the next forward pass.
Training Guide, "Step 4": the momentum buffer is owner-only state.

Plumbing only: the assignment comes from the library (``dmuon_assign_owners``,
identical on every rank), the step from ``dmuon_step`` on the owned matrices,
and the broadcasts from ``torch.distributed`` (NCCL over NVLink between GPUs;
no library kernel ever reads another GPU's memory).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import torch

from . import _dtype_code, dmuon_assign_owners, dmuon_step


def owned_step(params: Sequence[torch.Tensor], grads: Sequence[Optional[torch.Tensor]],
               mom_bufs: Sequence[Optional[torch.Tensor]], *, lr: float = 0.02, momentum: float = 0.95,
               nesterov: bool = True, ns_steps: int = 5, coeffs=None, wd: float = 0.0, group=None,
               async_op: bool = False,
               local_step: Optional[Callable[[List[torch.Tensor], List[torch.Tensor], List[torch.Tensor]], None]] = None):
    """One Muon step with dedicated ownership over the ranks of ``group``.

    Every rank passes the same list of parameters (replicated, equal shapes);
    ``grads[i]`` and ``mom_bufs[i]`` are read only where this rank owns matrix i
    (``None`` elsewhere is fine).  The owner updates its matrices with
    ``dmuon_step`` (or ``local_step(params, grads, bufs)``, e.g. for a CPU test),
    then every parameter is broadcast from its owner.  Returns the assignment
    ``(owner_of, loads, imbalance)``, plus the broadcast handles when
    ``async_op`` (wait on them before the parameters are next read).
    """
    import torch.distributed as dist

    single = not (dist.is_available() and dist.is_initialized())
    world = 1 if single else dist.get_world_size(group)
    rank = 0 if single else dist.get_rank(group)
    shapes = [(p.shape[0], p.shape[1], _dtype_code(p)) for p in params]
    owner_of, loads, imbalance = dmuon_assign_owners(shapes, world)
    mine = [i for i, o in enumerate(owner_of) if o == rank]
    if any(grads[i] is None or mom_bufs[i] is None for i in mine):
        raise ValueError("an owned matrix needs its gradient and momentum buffer")
    if mine:
        ps = [params[i] for i in mine]
        gs = [grads[i] for i in mine]
        bs = [mom_bufs[i] for i in mine]
        if local_step is not None:
            local_step(ps, gs, bs)
        else:
            dmuon_step(ps, gs, bs, lr=lr, momentum=momentum, nesterov=nesterov, ns_steps=ns_steps,
                       coeffs=coeffs, wd=wd)
    handles = []
    for i, p in enumerate(params):
        if single:
            break
        src = owner_of[i] if group is None else dist.get_global_rank(group, owner_of[i])
        handles.append(dist.broadcast(p, src=src, group=group, async_op=True))
    if async_op:
        return (owner_of, loads, imbalance), handles
    for h in handles:
        h.wait()
    return owner_of, loads, imbalance
