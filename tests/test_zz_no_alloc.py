"""The allocation-free Newton-Schulz call against the oracle and its twin.

Some callers cannot allocate device memory: a framework whose caching
allocator already owns the device, or a loop that must not allocate after
start-up because cudaMalloc can synchronise the device.  dmuon_ns_noalloc
serves them from a fixed scratch array that the library reserves on each
device.  It runs the kernels of dmuon_ns in the same order, so these tests
check, call after call (the array keeps the previous call's contents), that
its result matches the fp64 oracle within the path's tolerance and equals
dmuon_ns bit for bit; that it still works when every workspace allocation of
the library fails and leaves the device's free memory unchanged; and that it
refuses matrices the array cannot hold.
"""
import numpy as np
import pytest
import torch

import newton_schulz_grad_b200 as nsg
from oracle import muon as om
from tests.gpu_util import bits, rel_fro, to64

pytestmark = pytest.mark.gpu
TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def seeded(shape, seed, dtype):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(*shape, generator=g).to(dtype).to("cuda")


def check_against_oracle_and_twin(X, steps=5, coeffs=None):
    got = torch.full_like(X, float("nan"))
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    nsg.dmuon_ns_noalloc(X, got, steps=steps, coeffs=coeffs, status=status)
    twin = torch.empty_like(X)
    nsg.dmuon_ns(X, twin, steps=steps, coeffs=coeffs)
    torch.cuda.synchronize()
    assert int(status.item()) == nsg.DMUON_OK
    assert np.array_equal(bits(got), bits(twin))
    c = None if coeffs is None else [tuple(float(np.float32(v)) for v in t) for t in coeffs]
    assert rel_fro(to64(got), om.newton_schulz(to64(X), steps, c)) < TOL[X.dtype]
    return got


@pytest.mark.parametrize("cases", [
    [((2048, 1024), torch.bfloat16), ((300, 129), torch.float32)],
    [((512, 768), torch.bfloat16), ((512, 768), torch.bfloat16)],
    [((32, 4096), torch.bfloat16), ((1000, 96), torch.bfloat16)],
    [((4096, 1024), torch.bfloat16), ((1024, 2048), torch.float32)],
], ids=["tc-then-ffma", "same-shape-twice", "thin-then-tall", "largest-then-fp32"])
def test_two_calls_in_a_row_match_oracle_and_dmuon_ns(cases):
    for k, (shape, dtype) in enumerate(cases):
        check_against_oracle_and_twin(seeded(shape, 100 + 17 * k + shape[0], dtype))


def test_custom_coefficients_and_no_status_word():
    X = seeded((256, 512), 5, torch.bfloat16)
    coeffs = [(3.0, -3.2, 1.2), (2.0, -1.5, 0.5), (1.5, -0.5, 0.0)]
    got = torch.empty_like(X)
    want = torch.empty_like(X)
    nsg.dmuon_ns_noalloc(X, got, steps=3, coeffs=coeffs)
    nsg.dmuon_ns(X, want, steps=3, coeffs=coeffs)
    torch.cuda.synchronize()
    assert np.array_equal(bits(got), bits(want))
    c32 = [tuple(float(np.float32(v)) for v in t) for t in coeffs]
    assert rel_fro(to64(got), om.newton_schulz(to64(X), 3, c32)) < TOL[torch.bfloat16]


def test_works_when_allocation_fails_and_allocates_nothing(monkeypatch):
    X = seeded((1024, 2048), 9, torch.bfloat16)
    first = check_against_oracle_and_twin(X)  # warm-up: kernels loaded, array looked up
    out = torch.empty_like(X)
    torch.cuda.synchronize()
    monkeypatch.setenv("DMUON_FAULT_INJECT", "alloc")
    # the library's own workspace path now fails ...
    with pytest.raises(nsg.DmuonError) as ei:
        nsg.dmuon_ns(X, torch.empty_like(X))
    assert ei.value.status == nsg.DMUON_ERR_OOM
    # ... and the allocation-free call does not go near it
    free_before, _ = torch.cuda.mem_get_info()
    nsg.dmuon_ns_noalloc(X, out)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before
    assert np.array_equal(bits(out), bits(first))


def test_rejects_matrices_beyond_the_scratch_array():
    X = torch.zeros(2048, 2048, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(X)
    with pytest.raises(nsg.DmuonError) as ei:
        nsg.dmuon_ns_noalloc(X, out)
    assert ei.value.status == nsg.DMUON_ERR_INVALID_ARG
    assert "bytes of scratch" in str(ei.value)
