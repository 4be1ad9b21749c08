"""Global p-norm gradient clipping on the GPU against the fp64 oracle.

DMuon Training Guide, "Gradient Clipping": the Muon gradients are clipped by
their global p-norm after the reduce and before momentum + Newton-Schulz.
The norm is compared with the oracle's fp64 norm (fp32 partials of 4096
elements, each a chain of at most 16 + 5 + 8 fp32 roundings, then a fixed-order
fp64 sum: relative error below 29 * 2^-24 ~ 1.7e-6, bounded here by 1e-5); the scaled values are compared bit for bit with
the fp32 rounding contract fl(g * fl32(coef)), with the coefficient the GPU
read back, and the coefficient itself with the oracle's to 1e-5.
"""
import math

import numpy as np
import pytest
import torch

import newton_schulz_grad_b200 as nsg
from oracle import emulate as em
from oracle import muon as om
from tests.gpu_util import bits, dtype_name, to64

pytestmark = pytest.mark.gpu

MIXED = [(64, 64), (100, 37), (4096, 11008), (257, 129), (1, 1), (33, 1000), (130, 136)]


def make_grads(shapes, dtype, seed, scale=1.0):
    gen = torch.Generator().manual_seed(seed)
    out = []
    for r, c in shapes:
        t = torch.randn(r, c, generator=gen) * scale
        out.append(t.to(dtype).cuda())
    return out


def check_clip(grads, max_norm, norm_type):
    before = [g.clone() for g in grads]
    total_dev = torch.zeros(1, dtype=torch.float64, device="cuda")
    nsg.dmuon_clip_grad_norm(grads, max_norm, norm_type, total_dev)
    torch.cuda.synchronize()
    _, total, coef = om.clip_grad_norm([to64(g) for g in before], max_norm, norm_type)
    got_total = float(total_dev.item())
    assert math.isclose(got_total, total, rel_tol=1e-5), (got_total, total)
    # the coefficient the kernel applied, recomputed from its own total as the
    # kernel does (fp64, rounded once to fp32)
    k = np.float32(min(1.0, max_norm / (got_total + om.CLIP_EPS)))
    assert math.isclose(float(k), coef, rel_tol=1e-5)
    for b, g in zip(before, grads):
        want = em.clip_scale_fp32(b.float().cpu().numpy(), float(k), dtype_name(b))
        nan = np.isnan(want)
        got = g.float().cpu().numpy()
        assert np.array_equal(np.isnan(got), nan)  # NaN payloads differ between CPU and GPU
        want_t = torch.from_numpy(np.where(nan, 0, want)).to(b.dtype)
        got_t = torch.from_numpy(np.where(nan, 0, got)).to(b.dtype)
        assert np.array_equal(bits(got_t), bits(want_t))
    return got_total, float(k)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("norm_type", [2.0, 1.0, float("inf")], ids=["l2", "l1", "linf"])
def test_clip_mixed_shapes(dtype, norm_type):
    grads = make_grads(MIXED, dtype, 11)
    total, k = check_clip(grads, 1.0, norm_type)
    assert k < 1.0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_clip_no_op_when_under_the_bound(dtype):
    grads = make_grads(MIXED[:4], dtype, 12, scale=1e-3)
    before = [bits(g) for g in grads]
    _, k = check_clip(grads, 1e6, 2.0)
    assert k == 1.0
    for b, g in zip(before, grads):
        assert np.array_equal(b, bits(g))


def test_clip_zero_gradients_and_zero_max_norm():
    grads = make_grads([(64, 128), (3, 5)], torch.float32, 13)
    check_clip(grads, 0.0, 2.0)
    assert all(float(g.abs().max()) == 0.0 for g in grads)
    zeros = [torch.zeros(8, 8, device="cuda"), torch.zeros(5, 3, device="cuda")]
    total, k = check_clip(zeros, 1.0, 2.0)
    assert total == 0.0 and k == 1.0


def test_clip_many_matrices_of_one_shape_spans_table_batches():
    # more than one launch table per class (tables hold 256 matrices)
    grads = make_grads([(16, 24)] * 300 + [(40, 8)] * 3, torch.bfloat16, 14)
    check_clip(grads, 2.0, 2.0)


def test_clip_unaligned_views_take_the_scalar_path():
    base = torch.randn(1, 64 * 37 + 3, device="cuda")
    g = base[0, 3:].view(64, 37)  # fp32 rows of 148 bytes, start 12 bytes off
    assert g.is_contiguous()
    check_clip([g], 0.5, 2.0)


def test_clip_deterministic():
    grads = make_grads([(1024, 2816), (300, 300)], torch.float32, 15)
    a = [g.clone() for g in grads]
    b = [g.clone() for g in grads]
    ta = torch.zeros(1, dtype=torch.float64, device="cuda")
    tb = torch.zeros(1, dtype=torch.float64, device="cuda")
    nsg.dmuon_clip_grad_norm(a, 1.0, 2.0, ta)
    nsg.dmuon_clip_grad_norm(b, 1.0, 2.0, tb)
    torch.cuda.synchronize()
    assert ta.item() == tb.item()
    for x, y in zip(a, b):
        assert np.array_equal(bits(x), bits(y))


# ------------------------------------------------ clipping fused into the step
import workloads  # noqa: E402


def _clone(ts):
    return [t.clone() for t in ts]


@pytest.mark.parametrize("norm_type", [2.0, float("inf")], ids=["l2", "linf"])
@pytest.mark.parametrize("name", ["small_layer_bf16", "single_256x512_f32"])
def test_step_clipped_equals_clip_then_step(name, norm_type, monkeypatch):
    # small workspace cap: several chunks, run overlapped on two streams
    monkeypatch.setenv("DMUON_WS_CAP_MB", "64")
    w = workloads.get(name)
    ps, gs, bs = workloads.make_all(w, "cuda")
    g_bits = [bits(g) for g in gs]
    # reference order of operations: clip in place, then the plain step
    p1, g1, b1 = _clone(ps), _clone(gs), _clone(bs)
    t1 = torch.zeros(1, dtype=torch.float64, device="cuda")
    if norm_type == 2.0:
        max_norm = 0.25 * float(sum(float(g.double().norm()) ** 2 for g in gs)) ** 0.5
    else:
        max_norm = 0.5 * max(float(g.abs().max()) for g in gs)
    nsg.dmuon_clip_grad_norm(g1, max_norm, norm_type, t1)
    nsg.dmuon_step(p1, g1, b1, lr=w.lr, momentum=w.momentum, nesterov=w.nesterov, wd=0.1)
    # fused
    p2, b2 = _clone(ps), _clone(bs)
    t2 = torch.zeros(1, dtype=torch.float64, device="cuda")
    nsg.dmuon_step(p2, gs, b2, lr=w.lr, momentum=w.momentum, nesterov=w.nesterov, wd=0.1,
                   max_norm=max_norm, norm_type=norm_type, total_norm=t2)
    torch.cuda.synchronize()
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    nsg.dmuon_release_workspace()
    assert t1.item() == t2.item()
    assert max_norm / t1.item() < 0.6  # clipping is active
    for a, b in zip(p1 + b1, p2 + b2):
        assert np.array_equal(bits(a), bits(b))
    # the fused step leaves the gradients untouched
    for before, g in zip(g_bits, gs):
        assert np.array_equal(before, bits(g))


@pytest.mark.parametrize("name", ["small_layer_bf16", "single_256x512_f32"])
def test_step_clipped_matches_oracle(name):
    w = workloads.get(name)
    ps, gs, bs = workloads.make_all(w, "cuda")
    p_old = [to64(p) for p in ps]
    g_h = [to64(g) for g in gs]
    b_h = [to64(b) for b in bs]
    max_norm = 0.5
    total = torch.zeros(1, dtype=torch.float64, device="cuda")
    nsg.dmuon_step(ps, gs, bs, lr=w.lr, momentum=w.momentum, nesterov=w.nesterov,
                   ns_steps=w.ns_steps, wd=w.wd, max_norm=max_norm, total_norm=total)
    torch.cuda.synchronize()
    clipped, want_total, coef = om.clip_grad_norm(g_h, max_norm, 2.0)
    assert coef < 1.0
    assert math.isclose(total.item(), want_total, rel_tol=1e-5)
    p_new, b_new, _ = om.muon_step(p_old, clipped, b_h, w.lr, w.momentum, w.nesterov,
                                   w.ns_steps, None, w.wd)
    for k in range(w.count):
        dn = dtype_name(ps[k])
        step = np.linalg.norm(p_new[k] - p_old[k])
        err = np.linalg.norm(to64(ps[k]) - p_new[k])
        tol_rel = 2e-2 if dn == "bf16" else 1e-4
        store = 2.0 ** -8 if dn == "bf16" else 1e-6
        assert err <= tol_rel * step + store * np.linalg.norm(p_new[k]), (k, err, step)
        # the buffer holds mu*buf + clipped g, rounded to its dtype
        berr = np.linalg.norm(to64(bs[k]) - b_new[k])
        assert berr <= (2.0 ** -8 if dn == "bf16" else 1e-6) * np.linalg.norm(b_new[k])


def test_clip_non_finite_gradients():
    for norm_type in (2.0, 1.0, float("inf")):
        # a NaN: total NaN and coefficient NaN, so every gradient becomes NaN,
        # in both dtypes (PyTorch's clip_grad_norm_; the oracle agrees)
        for dt in (torch.float32, torch.bfloat16):
            a = make_grads([(64, 96), (10, 10)], dt, 16)
            a[1][3, 4] = float("nan")
            _, want_total, want_coef = om.clip_grad_norm([to64(g) for g in a], 1.0, norm_type)
            assert math.isnan(want_total) and math.isnan(want_coef)
            t = torch.zeros(1, dtype=torch.float64, device="cuda")
            nsg.dmuon_clip_grad_norm(a, 1.0, norm_type, t)
            torch.cuda.synchronize()
            assert math.isnan(t.item())
            assert all(bool(torch.isnan(g).all()) for g in a)
        # an infinity: total inf, coefficient 0 (inf * 0 is NaN, the rest 0)
        b = make_grads([(64, 96), (10, 10)], torch.bfloat16, 17)
        b[0][5, 6] = float("inf")
        total, k = check_clip(b, 1.0, norm_type)
        assert math.isinf(total) and k == 0.0


# ------------------------------------------------------------- bucketed clip
def _bucket_set(seed):
    # Training Guide, "Fused CUDA clip for regular / Muon / AdamW": e.g. Muon
    # matrices, AdamW matrices and vectors, regular parameters, each a bucket
    gen = torch.Generator().manual_seed(seed)

    def t(shape, dtype, scale=1.0):
        return (torch.randn(*shape, generator=gen) * scale).to(dtype).cuda()
    return [
        [t((300, 700), torch.bfloat16), t((64, 64), torch.bfloat16), t((1, 1), torch.bfloat16)],
        [t((4096,), torch.float32), t((3, 5, 7), torch.float32, 10.0), t((129, 33), torch.bfloat16)],
        [],
        [t((2048, 1408), torch.bfloat16, 1e-4), t((17,), torch.float32, 1e-4)],
        [t((1000, 3), torch.float32, 3.0)],
    ]


def _as2d(g):
    return g.view(-1, g.shape[-1]) if g.dim() >= 2 else g.view(1, -1)


@pytest.mark.parametrize("seed", [0, 1])
def test_clip_buckets_equal_separate_clips_bit_for_bit(seed):
    max_norms = [1.0, 5.0, 1.0, 1e4, 0.5]
    norm_types = [2.0, float("inf"), 2.0, 1.0, 2.0]
    buckets = _bucket_set(30 + seed)
    sep = [[g.clone() for g in b] for b in buckets]
    before = [[to64(_as2d(g)) for g in b] for b in buckets]
    totals = torch.full((5,), -1.0, dtype=torch.float64, device="cuda")
    nsg.dmuon_clip_grad_norm_buckets(buckets, max_norms, norm_types, totals)
    want_totals = []
    for b, mx, nt in zip(sep, max_norms, norm_types):
        one = torch.zeros(1, dtype=torch.float64, device="cuda")
        nsg.dmuon_clip_grad_norm([_as2d(g) for g in b], mx, nt, one)
        want_totals.append(float(one.item()) if b else 0.0)
    torch.cuda.synchronize()
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    assert totals.cpu().tolist() == want_totals          # same reduction order: same bits
    for b, s in zip(buckets, sep):
        for g, h in zip(b, s):
            assert np.array_equal(bits(g), bits(h))
    # and each bucket against the oracle's separate clip
    got = om.clip_grad_norm_buckets(before, max_norms, norm_types)
    for k, (out, total, coef) in enumerate(got):
        assert math.isclose(float(totals[k].item()), total, rel_tol=1e-5, abs_tol=0.0)
        for g, w in zip(buckets[k], out):
            err = np.abs(to64(_as2d(g)) - w).max()
            assert err <= 2 ** -7 * np.abs(w).max() + 1e-30, (k, err)
    assert got[3][2] == 1.0 and got[0][2] < 1.0      # one bucket under its bound, one clipped


def test_clip_buckets_nan_stays_in_its_bucket():
    buckets = _bucket_set(40)
    buckets[1][2][5, 6] = float("nan")
    keep = [bits(g) for g in buckets[3]]
    totals = torch.zeros(5, dtype=torch.float64, device="cuda")
    nsg.dmuon_clip_grad_norm_buckets(buckets, [1.0] * 5, 2.0, totals)
    torch.cuda.synchronize()
    t = totals.cpu().tolist()
    assert math.isnan(t[1]) and all(math.isfinite(v) for k, v in enumerate(t) if k != 1)
    assert all(torch.isnan(g).all() for g in buckets[1])
    assert all(torch.isfinite(g).all() for k in (0, 3, 4) for g in buckets[k])
    assert all(np.array_equal(a, bits(g)) for a, g in zip(keep, buckets[3]))  # under its bound: unchanged


def test_clip_buckets_many_buckets_and_tables():
    # the largest bucket count, and a bucket spanning two launch tables
    gen = torch.Generator().manual_seed(41)
    buckets = [[(torch.randn(4, 8 + k % 5, generator=gen) * (1 + k)).cuda()] for k in range(127)]
    buckets.append([torch.randn(16, 24, generator=gen).cuda() for _ in range(300)])
    sep = [[g.clone() for g in b] for b in buckets]
    nsg.dmuon_clip_grad_norm_buckets(buckets, [1.0 + 0.01 * k for k in range(128)], 2.0)
    for k, b in enumerate(sep):
        nsg.dmuon_clip_grad_norm(b, 1.0 + 0.01 * k, 2.0)
    torch.cuda.synchronize()
    for b, s in zip(buckets, sep):
        assert all(np.array_equal(bits(g), bits(h)) for g, h in zip(b, s))
