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
