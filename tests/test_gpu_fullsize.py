"""Parity at the full benchmark sizes: the Llama-7B, Llama-3.2-3B and MoE sets.

Each whole set runs through one dmuon_step call, exactly as the benchmark
launches it; the oracle then recomputes sampled matrices of every launch class
(e.g. 4096x4096, 11008x4096 transposed, 4096x11008) in fp64 on the host.
"""
import numpy as np
import pytest
import torch

import newton_schulz_grad_b200 as nsg
import workloads
from oracle import emulate as em
from oracle import muon as om
from tests.gpu_util import to64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def full_step_sampled_parity(w, sample):
    ps, gs, bs = workloads.make_all(w, "cuda")
    saved = {i: (to64(ps[i]), gs[i].float().cpu().numpy(), bs[i].float().cpu().numpy())
             for i in sample}
    nsg.dmuon_step(ps, gs, bs, lr=w.lr, momentum=w.momentum, nesterov=w.nesterov,
                   ns_steps=w.ns_steps, wd=w.wd)
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    for i in sample:
        p0, g, b = saved[i]
        want_b, _ = em.momentum_fp32(b, g, w.momentum, w.nesterov, "bf16")
        assert np.array_equal(bs[i].float().cpu().numpy().view(np.uint32), want_b.view(np.uint32))
        p_new, _, _ = om.muon_step([p0], [g.astype(np.float64)], [b.astype(np.float64)], w.lr,
                                   w.momentum, w.nesterov, w.ns_steps, None, w.wd)
        got = to64(ps[i])
        step = np.linalg.norm(p_new[0] - p0)
        err = np.linalg.norm(got - p_new[0])
        assert err <= 2e-2 * step + 2 ** -8 * np.linalg.norm(p_new[0]), (i, err / step)
    # every parameter stayed finite
    for p in ps:
        assert torch.isfinite(p).all()


def test_llama7b_full_step_sampled_parity():
    w = workloads.get("llama_7b_bf16")
    sample = [1, 4, 6]  # k_proj (4096x4096), gate_proj (11008x4096), down_proj (4096x11008)
    sample += [w.count - 3]  # a last-layer gate_proj (last chunk of its class)
    # layer 16's v_proj and gate_proj: members 66 of 128 and 48 of 96 of their
    # classes, in the middle chunk of each (chunks of 26 and of 12)
    sample += [114, 116]
    full_step_sampled_parity(w, sample)


def test_llama3_2_3b_full_step_sampled_parity():
    # 196 matrices, wd = 0.1; q (3072^2), k (1024x3072), gate (8192x3072,
    # transposed), down (3072x8192), and the last layer's up_proj
    w = workloads.get("llama3_2_3b_bf16")
    full_step_sampled_parity(w, [0, 1, 4, 6, w.count - 2])


def test_moe_full_step_sampled_parity():
    # 248 matrices: expert gate (1408x2048) and down (2048x1408), the first and
    # last of the seed-chosen 1e-4-scaled matrices, a thin 32x4096 GateDelta
    # projection (clustered one-launch chain) and a tall 16384x2048 matrix
    w = workloads.get("moe_skewed_bf16")
    sk = workloads.skewed_indices(w)
    full_step_sampled_parity(w, sorted({0, 2, sk[0], sk[-1], 192, w.count - 1}))


@pytest.mark.parametrize("shape", [(16384, 24576), (24576, 16384)])
def test_large_diagonal_closed_form(shape):
    # X = [D | 0] (or its transpose) with D diagonal: every product stays
    # diagonal, so at any size NS(X) = diag(f^5(d_i / ||d||)) exactly in real
    # arithmetic, with f(s) = a s + b s^3 + c s^5, and exact zeros elsewhere.
    # 16384 x 24576 runs every tile of the CTA-pair kernels and the Gram-space
    # block (n >= 1.25 m).
    R, C = shape
    m = min(R, C)
    d = (1.0 + torch.arange(m, dtype=torch.float32) / m).to(torch.bfloat16)
    X = torch.zeros(R, C, dtype=torch.bfloat16, device="cuda")
    X.diagonal().copy_(d.cuda())
    out = torch.full_like(X, float("nan"))
    nsg.dmuon_ns(X, out, steps=5)
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    dd = d.double().numpy()
    s = dd / (np.linalg.norm(dd) + om.NORM_EPS)
    a, b, c = (float(np.float32(v)) for v in om.DEFAULT_COEFFS)
    for _ in range(5):
        s = a * s + b * s ** 3 + c * s ** 5
    got = out.diagonal().double().cpu().numpy()
    assert np.linalg.norm(got - s) / np.linalg.norm(s) < 2e-2
    total = float(out.double().pow(2).sum().item())
    assert abs(total - float(np.sum(got ** 2))) <= 1e-12 * total   # nothing off the diagonal
    assert torch.isfinite(out).all()


def _f5(s):
    a, b, c = (float(np.float32(v)) for v in om.DEFAULT_COEFFS)
    for _ in range(5):
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def _sumsq_rows(t, rows=2048):
    return sum(float((t[i:i + rows].float() ** 2).sum(dtype=torch.float64)) for i in range(0, t.shape[0], rows))


@pytest.mark.parametrize("shape", [(32768, 65535), (65535, 32768)])
def test_max_elements_step_diagonal_closed_form(shape):
    # The largest matrix the ABI takes (rows * cols < 2^31; 18 GiB of
    # workspace, over the default cap, so a chunk of its own), through a whole
    # dmuon_step: gradient [D | 0] (or its transpose), zero buffer and
    # parameter.  The buffer becomes the gradient bit for bit, x0 = bf16(g +
    # 0.95 g) stays diagonal, NS(x0) = diag(f^5(x0_i / ||x0||)) exactly in real
    # arithmetic, and p' = -fl32(lr 0.2 sqrt(max side)) NS(x0) with nothing off
    # the diagonal.  Runs the transposing momentum pass, every tile of the pair
    # kernels, the Gram-space block and the fused update (column writes of p
    # for the tall orientation) at the maximum size.
    R, C = shape
    m = min(R, C)
    d = (1.0 + torch.arange(m, dtype=torch.float32) / m).to(torch.bfloat16)
    g = torch.zeros(R, C, dtype=torch.bfloat16, device="cuda")
    g.diagonal().copy_(d.cuda())
    p = torch.zeros_like(g)
    buf = torch.zeros_like(g)
    lr = 0.02
    nsg.dmuon_step([p], [g], [buf], lr=lr, momentum=0.95, nesterov=True, ns_steps=5, wd=0.0)
    torch.cuda.synchronize()
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    assert torch.equal(buf.diagonal(), g.diagonal()) and _sumsq_rows(buf) == _sumsq_rows(g)
    dd = d.float().numpy()
    _, x0 = em.momentum_fp32(np.zeros_like(dd), dd, 0.95, True, "bf16")
    x0 = x0.astype(np.float64)
    s = x0 / (np.linalg.norm(x0) + om.NORM_EPS)
    want = -float(em.update_scale(lr, R, C)) * _f5(s)
    got = p.diagonal().double().cpu().numpy()
    assert np.linalg.norm(got - want) / np.linalg.norm(want) < 2e-2
    assert abs(_sumsq_rows(p) - float(np.sum(got ** 2))) <= 1e-9 * float(np.sum(got ** 2))
    nsg.dmuon_release_workspace()


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, 2e-2), (torch.float32, 1e-4)], ids=["bf16", "f32"])
@pytest.mark.parametrize("shape", [(1, 1 << 20), (1 << 20, 1)])
def test_longest_side_vector_closed_form(shape, dtype, tol):
    # A vector has one singular value, ||x|| / (||x|| + eps) ~ 1 after the
    # normalisation, so NS(x) = f^5(1) x / ||x|| (f^5(1) = 0.69644 for the
    # default coefficients); 2^20 is the longest side the ABI takes
    gen = torch.Generator().manual_seed(5)
    x = torch.randn(*shape, generator=gen).to(dtype)
    out = torch.empty_like(x).cuda()
    nsg.dmuon_ns(x.cuda(), out, steps=5)
    torch.cuda.synchronize()
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    xv = x.double().numpy().ravel()
    nx = np.linalg.norm(xv)
    want = _f5(nx / (nx + om.NORM_EPS)) * xv / nx
    got = out.double().cpu().numpy().ravel()
    assert np.linalg.norm(got - want) / np.linalg.norm(want) < tol
