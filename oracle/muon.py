"""Oracle: a plain, slow, obviously correct fp64 CPU Muon step.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py`` may import this module.
The product path (the CUDA library and its Python binding) never calls it,
and it shares no code with that path: no kernels, headers, helpers or table
generators.  It takes its inputs as plain arrays (fp64 copies of whatever the
device holds) and uses numpy matmul as its only library primitive.

What it computes, per matrix, in the order of the DMuon documentation
(Training Guide, "Step 4: Create Optimizer" and its "Hyperparameter Guide"
table; FAQ, "Why isn't DMuon just ZeRO-1?"):

1. momentum:   buf' = mu * buf + g
2. Nesterov:   x0 = g + mu * buf'   (nesterov=True, the recommended default)
               x0 = buf'            (nesterov=False)
3. orient:     X = x0^T if rows > cols else x0  (work over the smaller side)
4. normalise:  X = X / (||X||_F + eps)
5. ns_steps Gram Newton-Schulz iterations, each
               G = X X^T ;  X = a X + (b G + c G G) X   ( = p(G) X )
6. un-orient:  O = X^T if rows > cols else X
7. update:     p' = p (1 - lr wd) - lr * 0.2 sqrt(max(rows, cols)) * O

Readings taken where the pages are silent (each is listed in the design
notes of the repository):

* The pages print the Nesterov input ``grad + mu * buf`` only; the buffer
  recurrence is read as ``buf <- mu*buf + g`` and Nesterov uses the updated
  buffer.
* The pages print no Newton-Schulz coefficients (only that custom ones may be
  passed).  The default triple is the widely used quintic
  (3.4445, -4.7750, 2.0315) for every iteration; every function takes the
  coefficients as an argument.
* The normalisation epsilon (1e-7, added to the norm) is not on the pages.
* "gram" is named on the pages, not defined: read as recomputing
  G = X X^T every iteration over the smaller dimension and applying p(G) X.
* Weight decay uses the unscaled lr; the update uses the shape-scaled lr
  (Hyperparameter Guide, ``lr`` row: scaled by 0.2 * sqrt(max(m, n))).
  Both use the old parameter.
* Rows == cols: no transpose.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

# Reading (pages print none): the widely used quintic Muon coefficients.
DEFAULT_COEFFS: Tuple[float, float, float] = (3.4445, -4.7750, 2.0315)
# Reading (pages silent): epsilon added to the Frobenius norm.
NORM_EPS: float = 1e-7
# Training Guide, "Hyperparameter Guide": lr row, "0.2 * sqrt(max(m,n))".
LR_SHAPE_FACTOR: float = 0.2


def coeff_schedule(steps: int, coeffs=None) -> List[Tuple[float, float, float]]:
    """Per-iteration (a, b, c) list.

    ``coeffs`` is None (default triple every step), one triple (used every
    step) or a sequence of ``steps`` triples / a flat array of 3*steps values.
    """
    if coeffs is None:
        return [DEFAULT_COEFFS] * steps
    arr = np.asarray(coeffs, dtype=np.float64).reshape(-1)
    if arr.size == 3:
        t = tuple(float(v) for v in arr)
        return [t] * steps
    if arr.size != 3 * steps:
        raise ValueError("coeffs must hold 3 or 3*steps values")
    return [tuple(float(v) for v in arr[3 * k:3 * k + 3]) for k in range(steps)]


def momentum_update(buf: np.ndarray, g: np.ndarray, mu: float,
                    nesterov: bool) -> Tuple[np.ndarray, np.ndarray]:
    """Momentum buffer update and Newton-Schulz input.

    Training Guide, "Hyperparameter Guide" table: momentum 0.95 default,
    nesterov row "ns_input = grad + mu * buf".  Returns (buf', x0).
    """
    buf = np.asarray(buf, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    new_buf = mu * buf + g
    x0 = g + mu * new_buf if nesterov else new_buf
    return new_buf, x0


def orient(m: np.ndarray) -> Tuple[np.ndarray, bool]:
    """Work over the smaller dimension: transpose when rows > cols."""
    m = np.asarray(m, dtype=np.float64)
    if m.shape[0] > m.shape[1]:
        return m.T, True
    return m, False


def frobenius_normalize(x: np.ndarray, eps: float = NORM_EPS) -> np.ndarray:
    """X / (||X||_F + eps)."""
    x = np.asarray(x, dtype=np.float64)
    return x / (math.sqrt(float(np.sum(x * x))) + eps)


def gram_ns_iterations(x: np.ndarray, steps: int, coeffs=None) -> np.ndarray:
    """The Gram Newton-Schulz iterations on an oriented, normalised X (m <= n).

    Each iteration forms the Gram matrix over the smaller side and applies the
    quintic polynomial through it: G = X X^T, X <- a X + (b G + c G G) X.
    (DMuon FAQ, "What related work should I cite?": the default "gram"
    backend follows Gram Newton-Schulz; Training Guide, ns_steps row.)
    """
    x = np.asarray(x, dtype=np.float64)
    for a, b, c in coeff_schedule(steps, coeffs):
        g = x @ x.T
        x = a * x + (b * g + c * (g @ g)) @ x
    return x


def newton_schulz(m: np.ndarray, steps: int = 5, coeffs=None,
                  eps: float = NORM_EPS) -> np.ndarray:
    """Orthogonalised update O for one matrix (orient, normalise, iterate)."""
    x, transposed = orient(m)
    x = frobenius_normalize(x, eps)
    x = gram_ns_iterations(x, steps, coeffs)
    return x.T if transposed else x


def lr_scale(rows: int, cols: int) -> float:
    """Shape-aware Muon lr factor 0.2 * sqrt(max(m, n)) (Hyperparameter Guide, lr row)."""
    return LR_SHAPE_FACTOR * math.sqrt(max(rows, cols))


def apply_update(p: np.ndarray, o: np.ndarray, lr: float, wd: float) -> np.ndarray:
    """p' = p (1 - lr wd) - lr * 0.2 sqrt(max(m,n)) * O (decoupled decay, old p)."""
    p = np.asarray(p, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    r, c = p.shape
    return p * (1.0 - lr * wd) - (lr * lr_scale(r, c)) * o


def muon_step(params: Sequence[np.ndarray], grads: Sequence[np.ndarray],
              bufs: Sequence[np.ndarray], lr: float = 0.02, momentum: float = 0.95,
              nesterov: bool = True, ns_steps: int = 5, coeffs=None, wd: float = 0.0,
              eps: float = NORM_EPS):
    """One Muon step over a list of 2D matrices, each independently.

    Training Guide, "Step 4": Group 0 (dedicated params) runs momentum + NS +
    update.  Returns (params', bufs', updates O), all fp64.
    """
    out_p, out_b, out_o = [], [], []
    for p, g, b in zip(params, grads, bufs):
        nb, x0 = momentum_update(b, g, momentum, nesterov)
        o = newton_schulz(x0, ns_steps, coeffs, eps)
        out_p.append(apply_update(p, o, lr, wd))
        out_b.append(nb)
        out_o.append(o)
    return out_p, out_b, out_o


# Reading (the Training Guide's "Gradient Clipping" section names global p-norm
# clipping of the Muon gradients, gives DMuon's clip the name and max_norm
# argument of PyTorch's clip_grad_norm_ and uses the two side by side):
# PyTorch's formula, 1e-6 added to the norm, coefficient clamped to 1 by a
# clamp that keeps a NaN.
CLIP_EPS: float = 1e-6


def clip_grad_norm(grads: Sequence[np.ndarray], max_norm: float, norm_type: float = 2.0):
    """Global p-norm clipping of a list of gradients.

    total = (sum_i sum |g|^p)^(1/p) (p = inf: max |g|); coef = clamp(max_norm /
    (total + 1e-6), max=1), NaN when total is NaN (so every gradient becomes
    NaN, as with PyTorch's clip_grad_norm_; the returned total is what a
    caller checks for non-finite values); returns (clipped gradients, total,
    coef).  Training Guide, "Gradient Clipping": after the reduce, before
    momentum + Newton-Schulz.
    """
    gs = [np.asarray(g, dtype=np.float64) for g in grads]
    if norm_type == float("inf"):
        # np.max keeps a NaN wherever it sits (Python's max would drop it)
        per = [np.max(np.abs(g)) for g in gs if g.size]
        total = float(np.max(per)) if per else 0.0
    else:
        p = float(norm_type)
        total = sum(float(np.sum(np.abs(g) ** p)) for g in gs) ** (1.0 / p)
    coef = max_norm / (total + CLIP_EPS)
    if not math.isnan(coef):
        coef = min(1.0, coef)
    with np.errstate(invalid="ignore"):
        return [g * coef for g in gs], total, coef


def clip_grad_norm_buckets(buckets: Sequence[Sequence[np.ndarray]], max_norms: Sequence[float],
                           norm_types: Sequence[float]):
    """Several independent clips at once.

    Training Guide, "Fused CUDA clip for regular / Muon / AdamW": when several
    gradient groups (buckets) are clipped together, each bucket keeps the
    semantics of its own clip: bucket k is clipped by the global
    norm_types[k]-norm of its gradients alone, with max_norms[k], exactly as
    clip_grad_norm clips that list.  An empty bucket has total 0.  Returns one
    (clipped gradients, total, coef) per bucket.
    """
    if not (len(buckets) == len(max_norms) == len(norm_types)):
        raise ValueError("one max_norm and one norm_type per bucket")
    return [clip_grad_norm(b, float(mx), float(nt)) for b, mx, nt in zip(buckets, max_norms, norm_types)]


def shape_groups(shapes: Sequence[Tuple[int, int, int]]):
    """Partition matrices by (rows, cols, dtype).

    Group ids are given in order of first appearance; the execution order is
    the concatenation of the groups, members in ascending index.  Returns
    (group_of, order, num_groups).
    """
    ids = {}
    group_of = []
    members: List[List[int]] = []
    for i, key in enumerate(shapes):
        key = tuple(int(v) for v in key)
        if key not in ids:
            ids[key] = len(members)
            members.append([])
        gid = ids[key]
        group_of.append(gid)
        members[gid].append(i)
    order = [i for grp in members for i in grp]
    return group_of, order, len(members)


def ns_iteration_flops(rows: int, cols: int) -> float:
    """Flops of one Gram Newton-Schulz iteration on one matrix: 3 m^2 n + m^3
    (m = min side, n = max side; one triangle of each symmetric product)."""
    m, n = float(min(rows, cols)), float(max(rows, cols))
    return 3.0 * m * m * n + m * m * m


def assign_owners(shapes: Sequence[Tuple[int, int]], world: int):
    """Dedicated ownership: every matrix to one rank, loads balanced.

    DMuon FAQ, "Why isn't DMuon just ZeRO-1?": one rank owns the whole matrix and
    runs Newton-Schulz on it, the others receive the updated parameter;
    Training Guide, "Verify Parameter Assignment": the assignment is reported
    with per-rank loads and an imbalance figure.  Reading (the pages give no
    rule): the load of a matrix is its Newton-Schulz flops per iteration; the
    matrices are taken from the most expensive down (equal costs: lower index
    first) and each goes to the rank with the least load so far (equal loads:
    lower rank); imbalance = max load / mean load - 1.  Returns (owner_of,
    loads, imbalance).
    """
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = [ns_iteration_flops(r, c) for r, c in shapes]
    order = sorted(range(len(shapes)), key=lambda i: (-cost[i], i))
    loads = [0.0] * world
    owner_of = [0] * len(shapes)
    for i in order:
        r = min(range(world), key=lambda k: (loads[k], k))
        owner_of[i] = r
        loads[r] += cost[i]
    mean = sum(loads) / world
    imbalance = (max(loads) / mean - 1.0) if mean > 0 else 0.0
    return owner_of, loads, imbalance
