"""GPU tests of the individual kernels, through the C ABI.

* gram / gram_poly / poly_apply (tcgen05 for bf16, FFMA for fp32) against an
  fp64 product of the same inputs, at sizes spanning several 128x256 tiles
  with ragged edges in every dimension;
* momentum and update stages bit for bit against the fp32 rounding-contract
  emulation.
"""
import numpy as np
import pytest
import torch

import newton_schulz_grad_b200 as nsg
from oracle import emulate as em
from tests.gpu_util import bits, rel_fro, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def rnd(shape, seed, dtype, scale=1.0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(dtype).to(DEV)


# bf16 output rounding (2^-9 relative per element) dominates; fp32 accumulation
TOL = {torch.bfloat16: 6e-3, torch.float32: 1e-5}
SHAPES = [(1, 64, 64), (3, 200, 328), (2, 384, 1000), (1, 136, 2056), (2, 520, 520), (1, 8, 24)]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("b,m,n", SHAPES)
def test_gram(dtype, b, m, n):
    X = rnd((b, m, n), 1 + m + n, dtype)
    G = torch.full((b, m, m), float("nan"), dtype=dtype, device=DEV)
    nsg.dmuon_gram(X, G, alpha=0.75)
    torch.cuda.synchronize()
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    x = to64(X)
    want = 0.75 * np.einsum("bik,bjk->bij", x, x)
    got = to64(G)
    assert np.isfinite(got).all()
    for i in range(b):
        assert rel_fro(got[i], want[i]) < TOL[dtype]
    # one triangle computed, the other mirrored: exactly symmetric
    assert np.array_equal(bits(G), bits(G.transpose(1, 2)))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("b,m", [(1, 64), (3, 200), (2, 384), (1, 520), (2, 8)])
def test_gram_poly(dtype, b, m):
    X = rnd((b, m, m + 40), 7 + m, torch.float32) / np.sqrt(m)
    Gs = (X @ X.transpose(1, 2))
    G = ((Gs + Gs.transpose(1, 2)) / 2).to(dtype).contiguous()
    G = torch.maximum(G, G.transpose(1, 2)).contiguous()  # exactly symmetric after rounding
    P = torch.full((b, m, m), float("nan"), dtype=dtype, device=DEV)
    nsg.dmuon_gram_poly(G, P, b=-4.775, c=2.0315)
    torch.cuda.synchronize()
    g = to64(G)
    want = -4.775 * g + 2.0315 * np.einsum("bik,bkj->bij", g, g)
    got = to64(P)
    for i in range(b):
        assert rel_fro(got[i], want[i]) < TOL[dtype]
    assert np.array_equal(bits(P), bits(P.transpose(1, 2)))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("b,m,n", SHAPES)
@pytest.mark.parametrize("symmetric", [True, False])
def test_poly_apply(dtype, b, m, n, symmetric):
    P = rnd((b, m, m), 3 + m, torch.float32) / np.sqrt(m)
    if symmetric:
        P = (P + P.transpose(1, 2)) / 2
    P = P.to(dtype).contiguous()
    X = rnd((b, m, n), 5 + n, dtype)
    Y = torch.full((b, m, n), float("nan"), dtype=dtype, device=DEV)
    nsg.dmuon_poly_apply(P, X, Y, a=3.4445, alpha=0.5)
    torch.cuda.synchronize()
    p, x = to64(P), to64(X)
    want = 0.5 * (3.4445 * x + np.einsum("bik,bkj->bij", p, x))
    got = to64(Y)
    for i in range(b):
        assert rel_fro(got[i], want[i]) < TOL[dtype]


def test_gram_padded_leading_dimension():
    # ld larger than the row: pad columns must be ignored
    base = rnd((2, 136, 264), 11, torch.bfloat16)
    X = base[:, :, :250]
    G = torch.zeros((2, 136, 144), dtype=torch.bfloat16, device=DEV)[:, :, :136]
    nsg.dmuon_gram(X, G)
    torch.cuda.synchronize()
    x = to64(X)
    want = np.einsum("bik,bjk->bij", x, x)
    got = to64(G)
    for i in range(2):
        assert rel_fro(got[i], want[i]) < 6e-3


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", [(1, 1), (7, 13), (64, 64), (100, 300), (300, 100), (257, 129)])
@pytest.mark.parametrize("nesterov", [True, False])
def test_momentum_bit_exact(dtype, shape, nesterov):
    g = rnd(shape, 21, dtype)
    buf = rnd(shape, 22, dtype, 0.5)
    x0 = torch.empty_like(g)
    sumsq = torch.zeros(1, dtype=torch.float64, device=DEV)
    want_b, want_x = em.momentum_fp32(buf.float().cpu().numpy(), g.float().cpu().numpy(), 0.95,
                                      nesterov, "bf16" if dtype == torch.bfloat16 else "f32")
    nsg.dmuon_momentum(buf, g, x0, momentum=0.95, nesterov=nesterov, sumsq=sumsq)
    torch.cuda.synchronize()
    assert np.array_equal(buf.float().cpu().numpy().view(np.uint32), want_b.view(np.uint32))
    assert np.array_equal(x0.float().cpu().numpy().view(np.uint32), want_x.view(np.uint32))
    ref = float(np.sum(want_x.astype(np.float64) ** 2))
    assert abs(float(sumsq.item()) - ref) <= 1e-6 * ref + 1e-30


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", [(1, 1), (7, 13), (64, 64), (100, 300), (300, 100), (257, 129)])
@pytest.mark.parametrize("wd", [0.0, 0.1])
def test_update_bit_exact(dtype, shape, wd):
    p = rnd(shape, 31, dtype, 0.02)
    o = rnd(shape, 32, dtype, 0.05)
    want = em.update_fp32(p.float().cpu().numpy(), o.float().cpu().numpy(), 0.02, wd,
                          "bf16" if dtype == torch.bfloat16 else "f32")
    nsg.dmuon_update(p, o, lr=0.02, wd=wd)
    torch.cuda.synchronize()
    assert np.array_equal(p.float().cpu().numpy().view(np.uint32), want.view(np.uint32))
