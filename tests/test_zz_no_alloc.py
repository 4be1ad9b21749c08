"""The allocation-free Newton-Schulz call against the regular one.

Some callers cannot allocate device memory: a framework whose caching
allocator already owns the device, or a loop that must not allocate after
start-up because cudaMalloc can synchronise the device.  dmuon_ns_noalloc
serves them from a fixed scratch array that the library reserves on each
device; these tests check that it gives the same results as dmuon_ns, call
after call (the array keeps the previous call's contents), and that it
refuses matrices the array cannot hold.
"""
import numpy as np
import pytest
import torch

import newton_schulz_grad_b200 as nsg
from tests.gpu_util import rel_fro, to64

pytestmark = pytest.mark.gpu
TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def seeded(shape, seed, dtype):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(*shape, generator=g).to(dtype).to("cuda")


@pytest.mark.parametrize("cases", [
    [((2048, 1024), torch.bfloat16), ((300, 129), torch.float32)],
    [((512, 768), torch.bfloat16), ((512, 768), torch.bfloat16)],
    [((32, 4096), torch.bfloat16), ((1000, 96), torch.bfloat16)],
], ids=["tc-then-ffma", "same-shape-twice", "thin-then-tall"])
def test_two_calls_in_a_row_match_dmuon_ns(cases):
    for k, (shape, dtype) in enumerate(cases):
        X = seeded(shape, 100 + 17 * k + shape[0], dtype)
        want = torch.empty_like(X)
        nsg.dmuon_ns(X, want, steps=5)
        got = torch.full_like(X, float("nan"))
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        nsg.dmuon_ns_noalloc(X, got, steps=5, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == nsg.DMUON_OK
        assert np.isfinite(to64(got)).all()
        assert rel_fro(to64(got), to64(want)) < TOL[dtype]


def test_custom_coefficients_and_no_status_word():
    X = seeded((256, 512), 5, torch.bfloat16)
    coeffs = [(3.0, -3.2, 1.2), (2.0, -1.5, 0.5), (1.5, -0.5, 0.0)]
    want = torch.empty_like(X)
    got = torch.empty_like(X)
    nsg.dmuon_ns(X, want, steps=3, coeffs=coeffs)
    nsg.dmuon_ns_noalloc(X, got, steps=3, coeffs=coeffs)
    torch.cuda.synchronize()
    assert rel_fro(to64(got), to64(want)) < TOL[torch.bfloat16]


def test_rejects_matrices_beyond_the_scratch_array():
    X = torch.zeros(2048, 2048, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(X)
    with pytest.raises(nsg.DmuonError) as ei:
        nsg.dmuon_ns_noalloc(X, out)
    assert ei.value.status == nsg.DMUON_ERR_INVALID_ARG
    assert "bytes of scratch" in str(ei.value)
