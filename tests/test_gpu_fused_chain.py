"""The whole Newton-Schulz chain of a chunk as one persistent launch.

On the tensor-core path each chunk's chain (every gram, polynomial /
Gram-space product and apply, the parameter update of the last apply
included) runs as one launch whose tiles wait on per-matrix counters instead
of kernel boundaries.  It computes the same tiles with the same epilogues as
one launch per product (DMUON_FUSED_CHAIN=0), so the results must be equal bit
for bit; they must also match the fp64 oracle.  Its dependency waits are
bounded: a dependency that is never met ends in DMUON_ERR_TIMEOUT with the
context still usable; and two chains on two streams at once (whose CTAs
compete for the SMs) must still finish with the bits of a serial run.
"""
import numpy as np
import pytest
import torch

import newton_schulz_grad_b200 as nsg
import workloads
from oracle import muon as om
from tests.gpu_util import bits, rel_fro, to64

pytestmark = pytest.mark.gpu


def seeded(shape, seed, scale=1.0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16).to("cuda")


def ns_both(X, monkeypatch, steps=5, coeffs=None):
    monkeypatch.setenv("DMUON_FUSED_CHAIN", "1")  # fused even where the default would not
    fused = torch.empty_like(X)
    nsg.dmuon_ns(X, fused, steps=steps, coeffs=coeffs)
    monkeypatch.setenv("DMUON_FUSED_CHAIN", "0")
    split = torch.empty_like(X)
    nsg.dmuon_ns(X, split, steps=steps, coeffs=coeffs)
    monkeypatch.delenv("DMUON_FUSED_CHAIN")
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    return fused, split


@pytest.mark.parametrize("shape", [(1024, 1024), (1024, 2816), (2816, 1024), (1408, 2048), (300, 700),
                                   (520, 300), (4096, 4096), (256, 6000)],
                         ids=lambda s: f"{s[0]}x{s[1]}")
def test_fused_chain_equals_product_launches_and_oracle(shape, monkeypatch):
    X = seeded(shape, shape[0] + 3 * shape[1])
    fused, split = ns_both(X, monkeypatch)
    assert np.array_equal(bits(fused), bits(split))
    assert rel_fro(to64(fused), om.newton_schulz(to64(X), 5)) < 2e-2


@pytest.mark.parametrize("mode", ["0", "1", "2"])
@pytest.mark.parametrize("steps", [1, 2, 3, 6])
def test_fused_chain_every_block_schedule(steps, mode, monkeypatch):
    # per-iteration form (0), Gram-space tail (1), blocks of 2, 3, 3 (2)
    monkeypatch.setenv("DMUON_GRAM_BLOCKS", mode)
    X = seeded((512, 1536), 40 + steps)
    coeffs = [(3.4445, -4.7750, 2.0315), (2.5, -2.0, 0.6), (1.5, -0.5, 0.0)] * 2
    fused, split = ns_both(X, monkeypatch, steps=steps, coeffs=coeffs[:steps])
    assert np.array_equal(bits(fused), bits(split))
    c32 = [tuple(float(np.float32(v)) for v in t) for t in coeffs[:steps]]
    assert rel_fro(to64(fused), om.newton_schulz(to64(X), steps, c32)) < 2e-2


@pytest.mark.parametrize("name,idx", [("small_layer_bf16", None), ("moe_skewed_bf16", [0, 1, 2, 3, 4, 5, 192, 240]),
                                      ("llama3_2_3b_bf16", [0, 1, 3, 4, 6, 7, 11])])
def test_fused_chain_steps_equal_product_launches(name, idx, monkeypatch):
    # whole steps (several chunks, transposed matrices, the fused update)
    w = workloads.get(name)
    sk = workloads.skewed_indices(w)
    idx = list(range(w.count)) if idx is None else idx
    monkeypatch.setenv("DMUON_WS_CAP_MB", "256")  # several chunks, overlapped
    runs = []
    for fused in ("1", "0"):
        monkeypatch.setenv("DMUON_FUSED_CHAIN", fused)
        mats = [workloads.make_matrix(w, i, "cuda", sk) for i in idx]
        ps, gs, bs = [m[0] for m in mats], [m[1] for m in mats], [m[2] for m in mats]
        nsg.dmuon_step(ps, gs, bs, wd=w.wd)
        assert nsg.dmuon_stream_status() == nsg.DMUON_OK
        runs.append([bits(t) for t in ps + bs])
    for a, b in zip(*runs):
        assert np.array_equal(a, b)


def test_fused_chain_dependency_wait_runs_out_and_recovers(monkeypatch):
    # a dependency nothing will meet: the bounded waits give up, the kernel
    # returns and the status word says so; the next call is unaffected
    X = seeded((1024, 2048), 77)
    out = torch.empty_like(X)
    monkeypatch.setenv("DMUON_FUSED_CHAIN", "1")
    monkeypatch.setenv("DMUON_FAULT_INJECT", "chain_wait")
    nsg.dmuon_ns(X, out)
    assert nsg.dmuon_stream_status() == nsg.DMUON_ERR_TIMEOUT
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK  # read and cleared
    monkeypatch.delenv("DMUON_FAULT_INJECT")
    fused, split = ns_both(X, monkeypatch)
    assert np.array_equal(bits(fused), bits(split))


def test_two_fused_chains_on_two_streams_at_once(monkeypatch):
    # both launches want every SM; tiles are claimed in order by running CTAs
    # only, so each finishes whatever share of the GPU it gets
    monkeypatch.setenv("DMUON_FUSED_CHAIN", "1")
    xs = [seeded((4096, 4096), 5 + k, 0.01) for k in range(2)]
    want = [torch.empty_like(x) for x in xs]
    for x, o in zip(xs, want):
        nsg.dmuon_ns(x, o)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in xs]
    got = [torch.empty_like(x) for x in xs]
    for _ in range(3):
        for x, o, s in zip(xs, got, streams):
            s.wait_stream(torch.cuda.current_stream())
            nsg.dmuon_ns(x, o, stream=s)
        torch.cuda.synchronize()
        for s in streams:
            assert nsg.dmuon_stream_status(s) == nsg.DMUON_OK
        for g, w in zip(got, want):
            assert np.array_equal(bits(g), bits(w))


# --------------------------------------------------------------- FFMA chains
def seeded_any(shape, seed, dtype):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(*shape, generator=g).to(dtype).to("cuda")


@pytest.mark.parametrize("shape,dtype", [((256, 512), torch.float32), ((40, 70), torch.float32),
                                         ((300, 129), torch.float32), ((1, 300), torch.float32),
                                         ((96, 200), torch.bfloat16), ((136, 130), torch.bfloat16),
                                         ((48, 30000), torch.bfloat16), ((1024, 640), torch.float32)],
                         ids=lambda v: str(v))
def test_fused_ffma_chain_equals_product_launches_and_oracle(shape, dtype, monkeypatch):
    # fp32 matrices, small near-square bf16 matrices (fp32 X) and thin bf16
    # matrices too wide for the clustered kernel all run the FFMA chain
    X = seeded_any(shape, 11 * shape[0] + shape[1], dtype)
    fused, split = ns_both(X, monkeypatch)
    assert np.array_equal(bits(fused), bits(split))
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    assert rel_fro(to64(fused), om.newton_schulz(to64(X), 5)) < tol


def test_fused_ffma_chain_steps_and_custom_coefficients(monkeypatch):
    X = seeded_any((256, 512), 3, torch.float32)
    coeffs = [(3.0, -3.2, 1.2), (2.0, -1.5, 0.5), (1.5, -0.5, 0.0)] * 6
    for steps in (1, 2, 7, 16, 17):  # 17 iterations: product by product
        fused, split = ns_both(X, monkeypatch, steps=steps, coeffs=coeffs[:steps])
        assert np.array_equal(bits(fused), bits(split))
    c32 = [tuple(float(np.float32(v)) for v in t) for t in coeffs[:7]]
    fused, _ = ns_both(X, monkeypatch, steps=7, coeffs=coeffs[:7])
    assert rel_fro(to64(fused), om.newton_schulz(to64(X), 7, c32)) < 1e-4


def test_fused_ffma_chain_wait_runs_out_and_recovers(monkeypatch):
    X = seeded_any((256, 512), 4, torch.float32)
    out = torch.empty_like(X)
    monkeypatch.setenv("DMUON_FAULT_INJECT", "chain_wait")
    nsg.dmuon_ns(X, out)
    assert nsg.dmuon_stream_status() == nsg.DMUON_ERR_TIMEOUT
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    monkeypatch.delenv("DMUON_FAULT_INJECT")
    fused, split = ns_both(X, monkeypatch)
    assert np.array_equal(bits(fused), bits(split))


def test_fused_ffma_chain_in_a_step(monkeypatch):
    # the single-matrix fp32 workload through dmuon_step: fused == per product
    w = workloads.get("single_256x512_f32")
    runs = []
    for fused in ("1", "0"):
        monkeypatch.setenv("DMUON_FUSED_CHAIN", fused)
        ps, gs, bs = workloads.make_all(w, "cuda")
        nsg.dmuon_step(ps, gs, bs, wd=0.1)
        assert nsg.dmuon_stream_status() == nsg.DMUON_OK
        runs.append([bits(t) for t in ps + bs])
    for a, b in zip(*runs):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("shape", [(1408, 2048), (2048, 1408), (300, 700), (4096, 4096), (1024, 2816)],
                         ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("fused", ["0", "1"])
def test_epilogue_width_gives_the_same_bits(shape, fused, monkeypatch):
    # four or eight epilogue warps drain the same accumulator columns with the
    # same arithmetic: the width may change the speed, never a bit
    monkeypatch.setenv("DMUON_FUSED_CHAIN", fused)
    X = seeded(shape, 7 * shape[0] + shape[1])
    p0 = seeded(shape, 11 + shape[0], 0.02)
    g = seeded(shape, 13 + shape[1])
    outs = []
    for width in ("4", "8"):
        monkeypatch.setenv("DMUON_EPI_WARPS", width)
        o = torch.empty_like(X)
        nsg.dmuon_ns(X, o)
        p, b = p0.clone(), torch.zeros_like(p0)
        nsg.dmuon_step([p], [g], [b], wd=0.1)     # the last apply fused with the update
        assert nsg.dmuon_stream_status() == nsg.DMUON_OK
        outs.append((bits(o), bits(p)))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("name,idx,cap", [("small_layer_bf16", None, None),
                                          ("small_layer_bf16", None, "64"),
                                          ("moe_skewed_bf16", [0, 1, 2, 3, 4, 5, 192, 193, 240, 241], "256"),
                                          ("single_256x512_f32", None, None)])
def test_two_chain_streams_give_the_same_bits(name, idx, cap, monkeypatch):
    # consecutive one-launch chains of a step run on two chain streams at
    # once; they read and write disjoint buffers, so one stream or two must
    # give the same bits (several chunks per class with the small cap)
    w = workloads.get(name)
    sk = workloads.skewed_indices(w)
    idx = list(range(w.count)) if idx is None else idx
    if cap:
        monkeypatch.setenv("DMUON_WS_CAP_MB", cap)
    runs = []
    for streams in ("2", "1"):
        monkeypatch.setenv("DMUON_CHAIN_STREAMS", streams)
        mats = [workloads.make_matrix(w, i, "cuda", sk) for i in idx]
        ps, gs, bs = [m[0] for m in mats], [m[1] for m in mats], [m[2] for m in mats]
        for _ in range(2):                      # two steps: the second reuses the buffers
            nsg.dmuon_step(ps, gs, bs, wd=w.wd)
        assert nsg.dmuon_stream_status() == nsg.DMUON_OK
        runs.append([bits(t) for t in ps + bs])
    for a, b in zip(*runs):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("fused", ["0", "1"])
@pytest.mark.parametrize("shape", [(4096, 4096), (1408, 2048), (2048, 1408), (1024, 2816), (300, 700), (520, 1300),
                                   (768, 768)], ids=lambda s: f"{s[0]}x{s[1]}")
def test_lower_stored_symmetric_matrices_give_the_same_bits(shape, fused, monkeypatch):
    # the chain stores G, p(G) and the Gram-space products as
    # their lower 256-column blocks and reads the upper part of each operand
    # as the transposed lower block; storing them in full must give the same
    # bits (same operand values, same products), in Newton-Schulz and in a
    # step with the fused update; per-product launches and the fused chain
    monkeypatch.setenv("DMUON_FUSED_CHAIN", fused)
    X = seeded(shape, 5 * shape[0] + shape[1])
    p0 = seeded(shape, 17 + shape[0], 0.02)
    g = seeded(shape, 19 + shape[1])
    outs = []
    for low in ("1", "0"):
        monkeypatch.setenv("DMUON_LOWER_STORE", low)
        o = torch.empty_like(X)
        nsg.dmuon_ns(X, o)
        p, b = p0.clone(), torch.zeros_like(p0)
        nsg.dmuon_step([p], [g], [b], wd=0.1)
        assert nsg.dmuon_stream_status() == nsg.DMUON_OK
        outs.append((bits(o), bits(p)))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    assert rel_fro(to64(o), om.newton_schulz(to64(X), 5)) < 2e-2
