"""Whole-path GPU parity against the fp64 oracle, through the C ABI.

Tolerances (per matrix, relative Frobenius):
* Newton-Schulz output O: 2e-2 for bf16 storage, 1e-4 for fp32;
* parameters: ||p_gpu - p_orc|| <= 2e-2 ||p_orc - p_old|| + 2^-8 ||p_orc||
  (the update is small next to p, and bf16 storage of p rounds at 2^-9);
* momentum buffers: bit for bit against the fp32 rounding-contract emulation.
"""
import os

import numpy as np
import pytest
import torch

import newton_schulz_grad_b200 as nsg
import workloads
from oracle import emulate as em
from oracle import muon as om
from tests.gpu_util import bits, dtype_name, rel_fro, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
NS_TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def lowrank_plus_noise(r, c, seed, dtype, rank=16, noise=1e-3):
    g = torch.Generator(device="cpu").manual_seed(seed)
    u, _ = torch.linalg.qr(torch.randn(r, min(rank, r, c), generator=g))
    v, _ = torch.linalg.qr(torch.randn(c, min(rank, r, c), generator=g))
    s = 1.0 / torch.arange(1, u.shape[1] + 1, dtype=torch.float32)
    m = (u * s) @ v.T + noise * torch.randn(r, c, generator=g)
    return m.to(dtype).to(DEV)


NS_CASES = [
    ((256, 512), torch.float32), ((40, 70), torch.float32), ((300, 129), torch.float32),
    ((256, 512), torch.bfloat16), ((1024, 1024), torch.bfloat16), ((2816, 1024), torch.bfloat16),
    ((1408, 2048), torch.bfloat16), ((2048, 1408), torch.bfloat16), ((32, 4096), torch.bfloat16),
    ((4096, 32), torch.bfloat16), ((96, 200), torch.bfloat16), ((200, 97), torch.bfloat16),
    ((65, 1000), torch.bfloat16), ((1, 300), torch.bfloat16), ((3, 5), torch.float32),
    ((130, 1001), torch.bfloat16), ((1001, 130), torch.bfloat16), ((77, 333), torch.float32),
]


@pytest.mark.parametrize("shape,dtype", NS_CASES, ids=lambda v: str(v))
def test_ns_matches_oracle(shape, dtype):
    X = lowrank_plus_noise(*shape, seed=shape[0] * 7 + shape[1], dtype=dtype)
    out = torch.empty_like(X)
    nsg.dmuon_ns(X, out, steps=5)
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    want = om.newton_schulz(to64(X), 5)
    assert rel_fro(to64(out), want) < NS_TOL[dtype]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_ns_custom_coefficients_and_zero_steps(dtype):
    X = lowrank_plus_noise(192, 320, 5, dtype)
    out = torch.empty_like(X)
    coeffs = [(3.0, -3.2, 1.2), (2.0, -1.5, 0.5), (1.5, -0.5, 0.0)]
    nsg.dmuon_ns(X, out, steps=3, coeffs=coeffs)
    c32 = [tuple(float(np.float32(v)) for v in t) for t in coeffs]
    assert rel_fro(to64(out), om.newton_schulz(to64(X), 3, c32)) < NS_TOL[dtype]
    nsg.dmuon_ns(X, out, steps=0)
    assert rel_fro(to64(out), om.newton_schulz(to64(X), 0)) < (4e-3 if dtype == torch.bfloat16 else 1e-6)


@pytest.mark.parametrize("mode", ["1", "2"])
@pytest.mark.parametrize("steps", [1, 2, 3, 4, 6, 12])
def test_ns_gram_space_blocks_match_oracle(steps, mode, monkeypatch):
    # wide bf16 matrices run their last two iterations as one Gram-space block
    # (mode 1, the default) or all of them in blocks of 2, 3, 3, ... (mode 2):
    # every block length and remainder appears across these steps
    monkeypatch.setenv("DMUON_GRAM_BLOCKS", mode)
    X = lowrank_plus_noise(300, 700, 21 + steps, torch.bfloat16, rank=32, noise=1e-2)
    out = torch.empty_like(X)
    coeffs = [(3.4445, -4.7750, 2.0315), (2.5, -2.0, 0.6), (1.5, -0.5, 0.0)] * 4
    nsg.dmuon_ns(X, out, steps=steps, coeffs=coeffs[:steps])
    c32 = [tuple(float(np.float32(v)) for v in t) for t in coeffs[:steps]]
    assert rel_fro(to64(out), om.newton_schulz(to64(X), steps, c32)) < 2e-2


def test_ns_gram_space_and_per_iteration_forms_agree(monkeypatch):
    X = lowrank_plus_noise(1024, 2816, 3, torch.bfloat16, rank=64, noise=1e-3)
    a, b = torch.empty_like(X), torch.empty_like(X)
    nsg.dmuon_ns(X, a)
    monkeypatch.setenv("DMUON_GRAM_BLOCKS", "0")
    nsg.dmuon_ns(X, b)
    torch.cuda.synchronize()
    want = om.newton_schulz(to64(X), 5)
    assert rel_fro(to64(a), want) < 2e-2 and rel_fro(to64(b), want) < 2e-2
    assert rel_fro(to64(a), to64(b)) < 3e-2


def test_ns_convergent_polynomial_reaches_polar_factor():
    X = lowrank_plus_noise(128, 256, 9, torch.float32, rank=128, noise=1e-2)
    out = torch.empty_like(X)
    nsg.dmuon_ns(X, out, steps=25, coeffs=(1.5, -0.5, 0.0))
    u, _, vt = np.linalg.svd(to64(X), full_matrices=False)
    assert rel_fro(to64(out), u @ vt) < 1e-4


def test_ns_transpose_equivariance_bf16():
    X = lowrank_plus_noise(384, 640, 3, torch.bfloat16)
    a, b = torch.empty_like(X), torch.empty_like(X.T.contiguous())
    nsg.dmuon_ns(X, a)
    nsg.dmuon_ns(X.T.contiguous(), b)
    torch.cuda.synchronize()
    # the tall input is transposed into the same oriented matrix: identical bits
    assert np.array_equal(bits(a), bits(b.T.contiguous()))


def test_ns_zero_matrix():
    X = torch.zeros(128, 256, dtype=torch.bfloat16, device=DEV)
    out = torch.full_like(X, 7.0)
    nsg.dmuon_ns(X, out)
    assert torch.count_nonzero(out).item() == 0


def run_step_check(w, idx=None):
    """dmuon_step over workload w (or the matrices idx of it) against the oracle."""
    sk = workloads.skewed_indices(w)
    idx = list(range(w.count)) if idx is None else idx
    mats = [workloads.make_matrix(w, i, DEV, sk) for i in idx]
    ps = [m[0] for m in mats]
    gs = [m[1] for m in mats]
    bs = [m[2] for m in mats]
    p_old = [to64(p) for p in ps]
    g_h = [g.float().cpu().numpy() for g in gs]
    b_h = [b.float().cpu().numpy() for b in bs]
    nsg.dmuon_step(ps, gs, bs, lr=w.lr, momentum=w.momentum, nesterov=w.nesterov,
                   ns_steps=w.ns_steps, wd=w.wd)
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    worst = 0.0
    for k in range(len(idx)):
        dn = dtype_name(ps[k])
        want_b, want_x = em.momentum_fp32(b_h[k], g_h[k], w.momentum, w.nesterov, dn)
        assert np.array_equal(bs[k].float().cpu().numpy().view(np.uint32), want_b.view(np.uint32))
        p_new, _, _ = om.muon_step([p_old[k]], [g_h[k].astype(np.float64)],
                                   [b_h[k].astype(np.float64)], w.lr, w.momentum, w.nesterov,
                                   w.ns_steps, None, w.wd)
        got = to64(ps[k])
        step = np.linalg.norm(p_new[0] - p_old[k])
        err = np.linalg.norm(got - p_new[0])
        tol_rel = 2e-2 if dn == "bf16" else 1e-4
        store = 2.0 ** -8 if dn == "bf16" else 1e-6
        assert err <= tol_rel * step + store * np.linalg.norm(p_new[0]), (idx[k], err, step)
        worst = max(worst, err / step)
    return worst


def test_step_single_matrix_f32():
    run_step_check(workloads.get("single_256x512_f32"))


def test_step_small_layer_bf16():
    run_step_check(workloads.get("small_layer_bf16"))


def test_step_llama3_2_3b_sampled():
    # one matrix of each shape class (q 3072^2, k 1024x3072, gate 8192x3072
    # transposed, down 3072x8192) plus a last-layer up_proj; wd = 0.1
    w = workloads.get("llama3_2_3b_bf16")
    run_step_check(w, [0, 1, 4, 6, w.count - 2])


def test_step_moe_sampled():
    w = workloads.get("moe_skewed_bf16")
    sk = workloads.skewed_indices(w)
    # two experts' matrices (one gate-shaped, one down-shaped), two skewed ones,
    # three GateDelta 32x4096 and one tall 16384x2048
    pick = sorted(set([0, 2, sk[0], sk[-1], 192, 200, 239, 240]))
    run_step_check(w, pick)


def test_step_batched_equals_solo_and_permuted():
    w = workloads.get("small_layer_bf16")
    mats = [workloads.make_matrix(w, i, DEV) for i in range(w.count)]

    def run(order):
        ps = [mats[i][0].clone() for i in order]
        gs = [mats[i][1].clone() for i in order]
        bs = [mats[i][2].clone() for i in order]
        nsg.dmuon_step(ps, gs, bs)
        torch.cuda.synchronize()
        return {i: (bits(p), bits(b)) for i, p, b in zip(order, ps, bs)}

    together = run(list(range(w.count)))
    perm = run([6, 2, 0, 5, 3, 1, 4])
    for i in range(w.count):
        solo = run([i])
        for res in (perm, solo):
            assert np.array_equal(res[i][0], together[i][0])
            assert np.array_equal(res[i][1], together[i][1])


def test_step_overlapped_equals_serial(monkeypatch):
    # several chunks (tiny workspace cap) run overlapped on two streams; the
    # result must be bitwise the one of the serial schedule
    w = workloads.get("small_layer_bf16")
    mats = [workloads.make_matrix(w, i, DEV) for i in range(w.count)]

    def run(env):
        for k, v in env.items():
            monkeypatch.setenv(k, v)
        ps = [m[0].clone() for m in mats]
        gs = [m[1].clone() for m in mats]
        bs = [m[2].clone() for m in mats]
        nsg.dmuon_step(ps, gs, bs, wd=0.1)
        torch.cuda.synchronize()
        assert nsg.dmuon_stream_status() == nsg.DMUON_OK
        return [bits(t) for t in ps + bs]

    serial = run({"DMUON_OVERLAP": "0", "DMUON_WS_CAP_MB": "64"})
    nsg.dmuon_release_workspace()
    over = run({"DMUON_OVERLAP": "1", "DMUON_WS_CAP_MB": "64"})
    nsg.dmuon_release_workspace()
    monkeypatch.delenv("DMUON_WS_CAP_MB")
    monkeypatch.delenv("DMUON_OVERLAP")
    assert all(np.array_equal(a, b) for a, b in zip(serial, over))


def test_step_zero_steps_and_no_nesterov():
    w = workloads.get("small_layer_bf16")
    ps, gs, bs = workloads.make_all(w, DEV)
    p_old = [to64(p) for p in ps]
    g_h = [g.float().cpu().numpy() for g in gs]
    b_h = [b.float().cpu().numpy() for b in bs]
    nsg.dmuon_step(ps, gs, bs, nesterov=False, ns_steps=0, wd=0.5, lr=0.01)
    torch.cuda.synchronize()
    for k in range(w.count):
        p_new, _, _ = om.muon_step([p_old[k]], [g_h[k]], [b_h[k]], 0.01, 0.95, False, 0, None, 0.5)
        err = np.linalg.norm(to64(ps[k]) - p_new[0])
        assert err <= 2e-2 * np.linalg.norm(p_new[0] - p_old[k]) + 2 ** -8 * np.linalg.norm(p_new[0])


def test_step_injected_allocation_failure_leaves_inputs(monkeypatch):
    w = workloads.get("small_layer_bf16")
    ps, gs, bs = workloads.make_all(w, DEV)
    before = [bits(t) for t in ps + bs]
    nsg.dmuon_release_workspace()
    monkeypatch.setenv("DMUON_FAULT_INJECT", "alloc")
    with pytest.raises(nsg.DmuonError) as ei:
        nsg.dmuon_step(ps, gs, bs)
    assert ei.value.status == nsg.DMUON_ERR_OOM
    monkeypatch.delenv("DMUON_FAULT_INJECT")
    torch.cuda.synchronize()
    after = [bits(t) for t in ps + bs]
    assert all(np.array_equal(a, b) for a, b in zip(before, after))


def test_step_empty_list():
    nsg.dmuon_step([], [], [])
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK


def test_bounded_device_wait_reports_timeout_and_context_survives():
    # a wait on a barrier that nothing arrives on gives up after 50 ms
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    nsg.dmuon_selftest_timeout(50000)
    assert nsg.dmuon_stream_status() == nsg.DMUON_ERR_TIMEOUT
    assert "ran out" in nsg.dmuon_get_last_error()
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK       # the word was cleared
    X = lowrank_plus_noise(256, 512, 3, torch.bfloat16)     # the context still works
    out = torch.empty_like(X)
    nsg.dmuon_ns(X, out)
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    assert rel_fro(to64(out), om.newton_schulz(to64(X), 5)) < 2e-2


@pytest.mark.parametrize("clip", [None, 0.5], ids=["plain", "clipped"])
@pytest.mark.parametrize("name", ["small_layer_bf16", "single_256x512_f32"])
def test_step_replays_from_a_cuda_graph(name, clip):
    # after one eager call on the capture stream (workspace and internal stream
    # exist) a step can be captured into a CUDA graph; replays give the eager
    # step's bits
    w = workloads.get(name)
    mats = [workloads.make_matrix(w, i, DEV) for i in range(w.count)]
    eager = [[t.clone() for t in m] for m in mats]
    graphed = [[t.clone() for t in m] for m in mats]
    scratch = [[t.clone() for t in m] for m in mats]

    def step(sets, stream=None):
        nsg.dmuon_step([m[0] for m in sets], [m[1] for m in sets], [m[2] for m in sets],
                       lr=w.lr, wd=0.05, stream=stream, max_norm=clip)

    step(eager)
    step(eager)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    step(scratch, stream=side)     # warm-up on the capture stream: allocations happen here
    side.synchronize()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        step(graphed, stream=side)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    for a, b in zip(eager, graphed):
        for x, y in zip(a, b):
            assert np.array_equal(bits(x), bits(y))


@pytest.mark.parametrize("shape,dtype", [((32, 4096), torch.bfloat16), ((4096, 32), torch.bfloat16),
                                         ((64, 1000), torch.bfloat16), ((16, 20000), torch.bfloat16),
                                         ((64, 9000), torch.bfloat16), ((64, 12000), torch.bfloat16),
                                         ((48, 4801), torch.float32), ((7, 300), torch.float32),
                                         ((1, 300), torch.bfloat16)], ids=str)
def test_thin_matrix_chain_matches_oracle_fused_and_unfused(shape, dtype, monkeypatch):
    # m <= 64 runs the whole chain in one clustered launch when the columns fit
    # the cluster's shared memory (64 x 12000 does not and falls back)
    X = lowrank_plus_noise(*shape, seed=sum(shape), dtype=dtype, rank=8, noise=1e-2)
    want = om.newton_schulz(to64(X), 5)
    fused = torch.empty_like(X)
    nsg.dmuon_ns(X, fused)
    monkeypatch.setenv("DMUON_SMALL_CHAIN", "0")
    plain = torch.empty_like(X)
    nsg.dmuon_ns(X, plain)
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    tol = NS_TOL[dtype]
    assert rel_fro(to64(fused), want) < tol
    assert rel_fro(to64(plain), want) < tol


@pytest.mark.parametrize("name,idx,env", [
    ("small_layer_bf16", None, {}),
    ("small_layer_bf16", None, {"DMUON_WS_CAP_MB": "64"}),        # several chunks, overlapped
    ("small_layer_bf16", None, {"DMUON_GRAM_BLOCKS": "2"}),        # blocks of 2 and 3
    ("small_layer_bf16", None, {"DMUON_GRAM_BLOCKS": "0"}),        # per-iteration form
    ("llama3_2_3b_bf16", [0, 1, 4, 6], {}),
    ("moe_skewed_bf16", [0, 2, 192, 240], {}),
], ids=["small", "small-overlap", "small-blocks2", "small-periter", "3b", "moe"])
def test_step_fused_update_equals_separate_pass(name, idx, env, monkeypatch):
    # the last apply's epilogue updates the parameters (default) or a separate
    # update kernel reads the stored result: same bits
    w = workloads.get(name)
    sk = workloads.skewed_indices(w)
    idx = list(range(w.count)) if idx is None else idx
    mats = [workloads.make_matrix(w, i, DEV, sk) for i in idx]
    for k, v in env.items():
        monkeypatch.setenv(k, v)

    def run(fused, steps=w.ns_steps):
        monkeypatch.setenv("DMUON_FUSED_UPDATE", "1" if fused else "0")
        ps = [m[0].clone() for m in mats]
        gs = [m[1].clone() for m in mats]
        bs = [m[2].clone() for m in mats]
        nsg.dmuon_step(ps, gs, bs, lr=w.lr, momentum=w.momentum, nesterov=w.nesterov,
                       ns_steps=steps, wd=0.1)
        torch.cuda.synchronize()
        assert nsg.dmuon_stream_status() == nsg.DMUON_OK
        nsg.dmuon_release_workspace()
        return [bits(t) for t in ps + bs]

    for steps in (w.ns_steps, 1, 2):
        a, b = run(True, steps), run(False, steps)
        assert all(np.array_equal(x, y) for x, y in zip(a, b)), steps


def test_step_fused_update_unaligned_parameter():
    # a parameter view 2 bytes off a 16-byte boundary takes the scalar path
    # of the fused epilogue (both orientations)
    for shape in ((256, 520), (520, 256)):
        gen = torch.Generator().manual_seed(7)
        base = (torch.randn(shape[0] * shape[1] + 1, generator=gen) * 0.02).to(torch.bfloat16).to(DEV)
        p = base[1:].view(*shape)
        g = torch.randn(*shape, generator=gen).to(torch.bfloat16).to(DEV)
        b = torch.zeros(*shape, dtype=torch.bfloat16, device=DEV)
        p_old = to64(p)
        head = bits(base[:1])
        nsg.dmuon_step([p], [g], [b], wd=0.1)
        torch.cuda.synchronize()
        want, _, _ = om.muon_step([p_old], [to64(g)], [np.zeros(shape)], 0.02, 0.95, True, 5, None, 0.1)
        err = np.linalg.norm(to64(p) - want[0])
        assert err <= 2e-2 * np.linalg.norm(want[0] - p_old) + 2 ** -8 * np.linalg.norm(want[0])
        assert np.array_equal(head, bits(base[:1]))  # the element before the view is untouched


def test_step_injected_launch_failure_is_ordered_and_recoverable(monkeypatch):
    # A launch failure part-way through an overlapped step: the status says so,
    # the parameters are untouched (the chain never ran), all of the call's
    # work is ordered before later work on the caller's stream, and the next
    # step gives the same bits as a step that never saw the failure.
    monkeypatch.setenv("DMUON_WS_CAP_MB", "64")
    w = workloads.get("small_layer_bf16")
    mats = [workloads.make_matrix(w, i, DEV) for i in range(w.count)]
    ref_p = [m[0].clone() for m in mats]
    ref_b = [m[2].clone() for m in mats]
    nsg.dmuon_step(ref_p, [m[1] for m in mats], ref_b)
    torch.cuda.synchronize()
    ps = [m[0].clone() for m in mats]
    bs = [m[2].clone() for m in mats]
    p_bits = [bits(p) for p in ps]
    monkeypatch.setenv("DMUON_FAULT_INJECT", "launch")
    with pytest.raises(nsg.DmuonError) as ei:
        nsg.dmuon_step(ps, [m[1] for m in mats], bs)
    assert ei.value.status == nsg.DMUON_ERR_CUDA and "injected" in str(ei.value)
    monkeypatch.delenv("DMUON_FAULT_INJECT")
    torch.cuda.current_stream().synchronize()
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    assert all(np.array_equal(a, bits(p)) for a, p in zip(p_bits, ps))
    # restore the buffers (the first chunk's momentum ran) and step again
    bs = [m[2].clone() for m in mats]
    nsg.dmuon_step(ps, [m[1] for m in mats], bs)
    torch.cuda.synchronize()
    assert all(np.array_equal(bits(a), bits(b)) for a, b in zip(ref_p + ref_b, ps + bs))
    nsg.dmuon_release_workspace()


def test_step_resumes_bitwise_in_a_new_process(tmp_path):
    # checkpoint / resume: the library keeps no state between steps beyond the
    # caller's parameters and momentum buffers, so two steps in one process
    # equal one step, torch.save, and a second step in a fresh process
    import subprocess
    import sys
    w = workloads.get("small_layer_bf16")
    ps, gs, bs = workloads.make_all(w, DEV)
    g2 = [torch.flip(g, dims=[0]).contiguous() for g in gs]
    nsg.dmuon_step(ps, gs, bs, wd=0.1)
    torch.cuda.synchronize()
    ck = tmp_path / "ck.pt"
    torch.save({"p": [p.cpu() for p in ps], "b": [b.cpu() for b in bs], "g2": [g.cpu() for g in g2]}, ck)
    nsg.dmuon_step(ps, g2, bs, wd=0.1)
    torch.cuda.synchronize()
    out = tmp_path / "out.pt"
    code = (
        "import torch, newton_schulz_grad_b200 as nsg\n"
        f"d = torch.load({str(ck)!r})\n"
        "ps = [t.cuda() for t in d['p']]; bs = [t.cuda() for t in d['b']]; gs = [t.cuda() for t in d['g2']]\n"
        "nsg.dmuon_step(ps, gs, bs, wd=0.1)\n"
        "torch.cuda.synchronize()\n"
        f"torch.save({{'p': [p.cpu() for p in ps], 'b': [b.cpu() for b in bs]}}, {str(out)!r})\n"
    )
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    subprocess.run([sys.executable, "-c", code], check=True, cwd=root, timeout=600)
    r = torch.load(out)
    assert all(np.array_equal(bits(a), bits(b)) for a, b in zip(ps + bs, r["p"] + r["b"]))


def test_step_with_nvtx_ranges_gives_the_same_bits(monkeypatch):
    w = workloads.get("small_layer_bf16")
    mats = [workloads.make_matrix(w, i, DEV) for i in range(w.count)]

    def run():
        ps = [m[0].clone() for m in mats]
        bs = [m[2].clone() for m in mats]
        nsg.dmuon_step(ps, [m[1] for m in mats], bs, max_norm=1.0)
        torch.cuda.synchronize()
        assert nsg.dmuon_stream_status() == nsg.DMUON_OK
        return [bits(t) for t in ps + bs]

    plain = run()
    monkeypatch.setenv("DMUON_NVTX", "1")
    with_ranges = run()
    assert all(np.array_equal(a, b) for a, b in zip(plain, with_ranges))


@pytest.mark.filterwarnings("ignore:The CUDA Graph is empty")
def test_step_refuses_to_grow_its_workspace_while_capturing():
    w = workloads.get("single_256x512_f32")
    ps, gs, bs = workloads.make_all(w, DEV)
    side = torch.cuda.Stream()          # never used: no workspace yet
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with pytest.raises(nsg.DmuonError) as ei:
        with torch.cuda.graph(g, stream=side):
            nsg.dmuon_step(ps, gs, bs, stream=side)
    assert ei.value.status == nsg.DMUON_ERR_INVALID_ARG and "capturing" in str(ei.value)
    torch.cuda.synchronize()
    nsg.dmuon_step(ps, gs, bs, stream=side)   # uncaptured, it allocates and runs
    side.synchronize()
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK


def test_concurrent_host_threads_on_their_own_streams():
    # two host threads step disjoint sets on their own streams at the same time
    # (the binding releases the GIL inside the library): each gets the bits of
    # a step run alone
    import threading
    w = workloads.get("small_layer_bf16")
    sets = [[[t.clone() for t in workloads.make_matrix(w, i, DEV)] for i in range(w.count)] for _ in range(2)]
    alone = [[[t.clone() for t in m] for m in s] for s in sets]
    for s in alone:
        nsg.dmuon_step([m[0] for m in s], [m[1] for m in s], [m[2] for m in s], wd=0.1)
    torch.cuda.synchronize()
    errors = []

    def worker(s):
        try:
            st = torch.cuda.Stream()
            st.wait_stream(torch.cuda.current_stream())
            for _ in range(1):
                nsg.dmuon_step([m[0] for m in s], [m[1] for m in s], [m[2] for m in s], wd=0.1, stream=st)
            st.synchronize()
        except Exception as exc:  # reported below
            errors.append(exc)

    threads = [threading.Thread(target=worker, args=(s,)) for s in sets]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    assert nsg.dmuon_stream_status() == nsg.DMUON_OK
    for s, a in zip(sets, alone):
        for m, n in zip(s, a):
            for x, y in zip(m, n):
                assert np.array_equal(bits(x), bits(y))
