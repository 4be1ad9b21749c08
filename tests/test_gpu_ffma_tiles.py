"""FFMA tile shapes and operand alignment give the same bits.

The FFMA kernels (fp32 matrices, small bf16 matrices whose X, G and p(G) stay
in fp32) sum every output element over k in ascending order, in blocks of
256, whatever the output tile: a chain too small to fill the GPU with
64 x 64 tiles runs 32 x 32 tiles, and DMUON_FFMA_TILE=64 / =32 forces either
shape, so both must give the same bits.  Operands move from global memory in
aligned 16-byte runs where the pointer, the leading dimension and the batch
stride allow, element by element otherwise: an operand that starts one
element past a 16-byte boundary, or whose rows are an odd number of elements
apart, must give the bits of an aligned copy.
"""
import numpy as np
import pytest
import torch

import newton_schulz_grad_b200 as nsg
from oracle import muon as om
from tests.gpu_util import bits, rel_fro, to64

pytestmark = pytest.mark.gpu


def seeded(shape, seed, dtype=torch.float32):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(*shape, generator=g).to(dtype).to("cuda")


@pytest.mark.parametrize("shape,dtype", [((256, 512), torch.float32), ((40, 70), torch.float32),
                                         ((300, 129), torch.float32), ((1, 300), torch.float32),
                                         ((97, 333), torch.float32), ((1024, 640), torch.float32),
                                         ((96, 200), torch.bfloat16), ((136, 130), torch.bfloat16),
                                         ((48, 30000), torch.bfloat16)],
                         ids=lambda v: str(v))
def test_ffma_tile_shape_gives_the_same_bits(shape, dtype, monkeypatch):
    X = seeded(shape, 5 * shape[0] + shape[1], dtype)
    outs = []
    for tile in ("64", "32"):
        monkeypatch.setenv("DMUON_FFMA_TILE", tile)
        o = torch.empty_like(X)
        nsg.dmuon_ns(X, o)
        assert nsg.dmuon_stream_status() == nsg.DMUON_OK
        outs.append(bits(o))
    assert np.array_equal(outs[0], outs[1])
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    assert rel_fro(to64(o), om.newton_schulz(to64(X), 5)) < tol


def test_ffma_tile_shape_in_a_batched_step(monkeypatch):
    # several fp32 matrices of one shape form one chunk; the whole step
    # (momentum, normalisation, chain, update) with either tile shape
    shapes = [(200, 328)] * 3 + [(256, 512)]
    runs = []
    for tile in ("64", "32"):
        monkeypatch.setenv("DMUON_FFMA_TILE", tile)
        ps = [seeded(s, 30 + i) * 0.02 for i, s in enumerate(shapes)]
        gs = [seeded(s, 60 + i) for i, s in enumerate(shapes)]
        bs = [seeded(s, 90 + i) * 0.01 for i, s in enumerate(shapes)]
        nsg.dmuon_step(ps, gs, bs, wd=0.1)
        assert nsg.dmuon_stream_status() == nsg.DMUON_OK
        runs.append([bits(t) for t in ps + bs])
    for a, b in zip(*runs):
        assert np.array_equal(a, b)


def offset_copy(t, shift, extra_cols):
    """t's values in a buffer where they start `shift` elements in and rows are
    cols + extra_cols apart (a strided view)."""
    b, r, c = t.shape
    ld = c + extra_cols
    buf = torch.full((shift + b * r * ld,), float("nan"), dtype=t.dtype, device=t.device)
    v = buf[shift:].view(b, r, ld)[:, :, :c]
    v.copy_(t)
    return v


@pytest.mark.parametrize("shift,extra", [(0, 2), (1, 2), (0, 1), (3, 6)])
def test_ffma_stage_calls_unaligned_operands(shift, extra):
    # fp32 stage calls run the FFMA kernels.  The contiguous operands: X rows
    # of 130 elements (not a multiple of 4: element by element), G, P and Y
    # of 72 (aligned runs); the views start `shift` elements in with rows
    # `extra` elements longer, so every operand changes between aligned runs
    # with a ragged tail and element-by-element loads
    B, m, n = 3, 72, 130
    X = seeded((B, m, n), 3)
    P = seeded((B, m, m), 4)
    G = torch.empty(B, m, m, device="cuda")
    nsg.dmuon_gram(X, G, alpha=0.5)
    Gv = offset_copy(torch.zeros_like(G), shift, extra)
    nsg.dmuon_gram(offset_copy(X, shift, extra), Gv, alpha=0.5)
    assert np.array_equal(bits(G), bits(Gv))
    Gs = (G + G.transpose(1, 2)) * 0.5
    Q = torch.empty_like(Gs)
    nsg.dmuon_gram_poly(Gs, Q, -1.5, 0.75)
    Qv = offset_copy(torch.zeros_like(Q), shift, extra)
    nsg.dmuon_gram_poly(offset_copy(Gs, shift, extra), Qv, -1.5, 0.75)
    assert np.array_equal(bits(Q), bits(Qv))
    Y = torch.empty_like(X)
    nsg.dmuon_poly_apply(P, X, Y, 1.25, 0.5)
    Yv = offset_copy(torch.zeros_like(Y), shift, extra)
    nsg.dmuon_poly_apply(offset_copy(P, shift, extra), offset_copy(X, shift, extra), Yv, 1.25, 0.5)
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    assert np.array_equal(bits(Y), bits(Yv))
    x, p, g = to64(X), to64(P), to64(Gs)
    assert rel_fro(to64(G), 0.5 * x @ x.transpose(0, 2, 1)) < 1e-5
    assert rel_fro(to64(Q), -1.5 * g + 0.75 * g @ g) < 1e-5
    assert rel_fro(to64(Y), 0.5 * (1.25 * x + p @ x)) < 1e-5
