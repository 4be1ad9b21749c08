"""Host-side tests of the C ABI: symbols, planning, validation (no GPU work)."""
import ctypes
import os
import random
import re

import pytest
import torch

import newton_schulz_grad_b200 as nsg
import workloads
from oracle import muon as om

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dmuon.h")
NO_GPU = not torch.cuda.is_available()


def declared_symbols():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"DMUON_API\s+[\w\s\*]+?\b(dmuon_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    syms = declared_symbols()
    assert len(syms) >= 15
    lib = nsg.library()
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) == set(nsg.EXPORTED)


def test_build_info_names_target():
    info = nsg.dmuon_build_info()
    assert "sm_100a" in info and "tcgen05" in info


@pytest.mark.parametrize("seed", range(20))
def test_plan_groups_matches_oracle(seed):
    rng = random.Random(seed)
    n = rng.randint(0, 60)
    shapes = [(rng.choice([1, 32, 1024, 2816]), rng.choice([1, 32, 1024]), rng.randint(0, 1))
              for _ in range(n)]
    assert nsg.dmuon_plan_groups(shapes) == om.shape_groups(shapes)


@pytest.mark.parametrize("w", workloads.WORKLOADS, ids=lambda w: w.name)
def test_plan_groups_on_workloads(w):
    code = 0 if w.dtype == "f32" else 1
    shapes = [(r, c, code) for r, c in w.shapes]
    g, order, k = nsg.dmuon_plan_groups(shapes)
    assert (g, order, k) == om.shape_groups(shapes)
    expect = {"single_256x512_f32": 1, "small_layer_bf16": 4, "llama3_2_3b_bf16": 4,
              "llama_7b_bf16": 3, "moe_skewed_bf16": 4}[w.name]
    assert k == expect


def test_launch_count_and_workspace_llama7b():
    w = workloads.get("llama_7b_bf16")
    shapes = [(r, c, 1) for r, c in w.shapes]
    # classes: 4096x4096 (128 matrices, 128 MiB of workspace each, one
    # iteration at a time) and 4096x11008 oriented (gate/up transposed + down:
    # 96 matrices; three iterations one at a time, then the last two as one
    # Gram-space block; five m x m slots: 340 MiB each).  Several chunks ->
    # overlapped execution with two buffers of half the 8 GiB cap: 5 chunks of
    # <= 26 and 8 chunks of 12.  Per chunk: momentum + norm (the update runs in
    # the last apply's epilogue), plus 3 per single iteration and gram + 5
    # products + apply for the block of two (chunks this large run one launch
    # per product)
    assert nsg.dmuon_step_launches(shapes, 5) == 5 * (2 + 15) + 8 * (2 + 9 + 7)
    os.environ["DMUON_GRAM_BLOCKS"] = "2"
    try:  # blocks of 2 and 3: gram + 5 products + apply, gram + 9 products + apply
        assert nsg.dmuon_step_launches(shapes, 5) == 5 * (2 + 15) + 8 * (2 + 7 + 11)
    finally:
        del os.environ["DMUON_GRAM_BLOCKS"]
    os.environ["DMUON_FUSED_UPDATE"] = "0"
    try:  # a separate update pass per chunk
        assert nsg.dmuon_step_launches(shapes, 5) == 5 * (3 + 15) + 8 * (3 + 9 + 7)
    finally:
        del os.environ["DMUON_FUSED_UPDATE"]
    ws = nsg.dmuon_workspace_bytes(shapes, 5)
    assert 5 << 30 < ws <= 8 << 30


def test_launch_count_fused_chains(monkeypatch):
    # small chunks fuse their whole chain into one launch; DMUON_FUSED_CHAIN=1
    # fuses every chain that can be (blocks of 2 and 3, 18 products, included),
    # =0 none
    w = workloads.get("small_layer_bf16")
    small = [(r, c, 1) for r, c in w.shapes]
    assert nsg.dmuon_step_launches(small, 5) == 3 * (2 + 1)  # three classes, one chunk each
    monkeypatch.setenv("DMUON_FUSED_CHAIN", "0")
    assert nsg.dmuon_step_launches(small, 5) == (2 + 15) + 2 * (2 + 9 + 7)  # 1024^2; 256x1024 and 1024x2816 with the tail
    w = workloads.get("llama_7b_bf16")
    shapes = [(r, c, 1) for r, c in w.shapes]
    monkeypatch.setenv("DMUON_FUSED_CHAIN", "1")
    assert nsg.dmuon_step_launches(shapes, 5) == 13 * (2 + 1)
    monkeypatch.setenv("DMUON_GRAM_BLOCKS", "2")
    assert nsg.dmuon_step_launches(shapes, 5) == 13 * (2 + 1)


def test_fused_chain_falls_back_where_products_disagree(monkeypatch):
    # m = 2100: the triangle products would take the one-CTA kernel and the
    # apply the CTA pair, so the chain runs product by product (same bits as
    # before); the per-iteration limit of the fused launch is 32 products
    assert nsg.dmuon_step_launches([(2100, 2100, 1)], 5) == 2 + 15
    assert nsg.dmuon_step_launches([(2048, 2048, 1)], 5) == 2 + 1
    assert nsg.dmuon_step_launches([(2048, 2048, 1)], 10) == 2 + 1
    assert nsg.dmuon_step_launches([(2048, 2048, 1)], 11) == 2 + 33


def test_overlap_can_be_disabled(monkeypatch):
    w = workloads.get("llama_7b_bf16")
    shapes = [(r, c, 1) for r, c in w.shapes]
    monkeypatch.setenv("DMUON_OVERLAP", "0")
    monkeypatch.setenv("DMUON_GRAM_BLOCKS", "0")
    assert nsg.dmuon_step_launches(shapes, 5) == 6 * (2 + 15)
    assert nsg.dmuon_workspace_bytes(shapes, 5) <= 8 << 30


def test_launch_count_thin_and_fp32_chunks(monkeypatch):
    # fp32 and thin bf16 classes keep the separate update; thin bf16 chains
    # (m <= 64) are one clustered launch, the other FFMA chains one fused launch
    # (up to 16 iterations, product by product beyond or with DMUON_FUSED_CHAIN=0)
    assert nsg.dmuon_step_launches([(256, 512, 0)], 5) == 3 + 1
    assert nsg.dmuon_step_launches([(100, 200, 1)], 5) == 3 + 1   # bf16, fp32 X
    assert nsg.dmuon_step_launches([(256, 512, 0)], 17) == 3 + 17 * 3
    monkeypatch.setenv("DMUON_FUSED_CHAIN", "0")
    assert nsg.dmuon_step_launches([(256, 512, 0)], 5) == 3 + 5 * 3
    monkeypatch.delenv("DMUON_FUSED_CHAIN")
    assert nsg.dmuon_step_launches([(32, 4096, 1)] * 3, 5) == 3 + 1
    assert nsg.dmuon_step_launches([(4096, 32, 1)], 5) == 3 + 1
    assert nsg.dmuon_step_launches([(32, 4096, 1)], 0) == 3
    assert nsg.dmuon_step_launches([(1024, 1024, 1)], 0) == 3


def _raw_step(count, params, grads, bufs, shapes, ns_steps=5, nesterov=1, lr=0.02):
    lib = nsg.library()
    vp = ctypes.c_void_p
    pa = (vp * max(1, len(params)))(*params)
    ga = (vp * max(1, len(grads)))(*grads)
    ba = (vp * max(1, len(bufs)))(*bufs)
    return lib.dmuon_step(pa, ga, ba, nsg._shape_array(shapes), count, lr, 0.95, nesterov,
                          ns_steps, None, 0.0, None)


def test_step_validation_errors():
    A = 1 << 40
    ok_shape = [(4, 8, 1)]
    assert _raw_step(-1, [A], [A + 4096], [A + 8192], ok_shape) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_step(0, [], [], [], []) == nsg.DMUON_OK
    assert _raw_step(1, [0], [A + 4096], [A + 8192], ok_shape) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_step(1, [A], [A + 4096], [A + 8192], [(0, 8, 1)]) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_step(1, [A], [A + 4096], [A + 8192], [(4, 8, 7)]) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_step(1, [A], [A + 4096], [A + 8192], [(1 << 21, 8, 1)]) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_step(1, [A], [A + 4096], [A + 8192], ok_shape, ns_steps=-1) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_step(1, [A], [A + 4096], [A + 8192], ok_shape, nesterov=2) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_step(1, [A], [A + 4096], [A + 8192], ok_shape, lr=float("nan")) == nsg.DMUON_ERR_INVALID_ARG
    # overlap: the grad starts inside the param (4*8*2 = 64 bytes)
    assert _raw_step(1, [A], [A + 32], [A + 8192], ok_shape) == nsg.DMUON_ERR_INVALID_ARG
    assert "overlap" in nsg.dmuon_get_last_error()
    # two matrices sharing a buffer
    assert _raw_step(2, [A, A + 100000], [A + 4096, A + 200000], [A + 8192, A + 8192],
                     ok_shape * 2) == nsg.DMUON_ERR_INVALID_ARG


def test_stage_validation_errors():
    lib = nsg.library()
    A = 1 << 40
    # bf16 stage calls need ld % 8 == 0 and 16-byte aligned pointers
    assert lib.dmuon_gram(A, A + (1 << 20), 1, 100, 100, 100, 100, 1.0, 1, None) == nsg.DMUON_ERR_INVALID_ARG
    assert lib.dmuon_gram(A + 2, A + (1 << 20), 1, 96, 96, 96, 96, 1.0, 1, None) == nsg.DMUON_ERR_INVALID_ARG
    assert lib.dmuon_gram(A, A + (1 << 20), 1, 96, 96, 64, 96, 1.0, 1, None) == nsg.DMUON_ERR_INVALID_ARG
    assert lib.dmuon_gram_poly(A, 0, 1, 96, 96, 96, 1.0, 1.0, 1, None) == nsg.DMUON_ERR_INVALID_ARG
    assert lib.dmuon_poly_apply(A, A, A, -1, 8, 8, 8, 8, 8, 1.0, 1.0, 1, None) == nsg.DMUON_ERR_INVALID_ARG
    assert lib.dmuon_ns_ex(A, A + 16, 4, 4, 5, None, 1, None) == nsg.DMUON_ERR_INVALID_ARG  # overlap
    assert lib.dmuon_ns_ex(A, A + 4096, 4, 4, -2, None, 1, None) == nsg.DMUON_ERR_INVALID_ARG
    assert lib.dmuon_momentum(A, A + 4096, A + 8192, 4, 4, 0.9, 3, 1, None, None) == nsg.DMUON_ERR_INVALID_ARG
    assert lib.dmuon_update(A, 0, 4, 4, 0.1, 0.0, 1, None) == nsg.DMUON_ERR_INVALID_ARG
    assert lib.dmuon_selftest_timeout(0, None) == nsg.DMUON_ERR_INVALID_ARG


@pytest.mark.skipif(not NO_GPU, reason="checks the no-device path")
def test_valid_call_without_device_reports_cuda_error():
    A = 1 << 40
    rc = _raw_step(1, [A], [A + 4096], [A + 8192], [(4, 8, 1)])
    assert rc in (nsg.DMUON_ERR_CUDA, nsg.DMUON_ERR_UNSUPPORTED)
    assert nsg.dmuon_get_last_error()


def _raw_clip(count, ptrs, shapes, max_norm=1.0, norm_type=2.0):
    lib = nsg.library()
    arr = (ctypes.c_void_p * max(1, len(ptrs)))(*ptrs)
    return lib.dmuon_clip_grad_norm(arr, nsg._shape_array(shapes), count, max_norm, norm_type, None, None)


def test_clip_validation_errors():
    A = 1 << 40
    ok = [(4, 8, 1)]
    assert _raw_clip(0, [], []) == nsg.DMUON_OK
    assert _raw_clip(-1, [A], ok) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_clip(1, [0], ok) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_clip(1, [A], [(4, 8, 5)]) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_clip(1, [A], [(0, 8, 1)]) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_clip(1, [A], ok, max_norm=float("nan")) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_clip(1, [A], ok, max_norm=-1.0) == nsg.DMUON_ERR_INVALID_ARG
    assert _raw_clip(1, [A], ok, norm_type=3.0) == nsg.DMUON_ERR_UNSUPPORTED
    assert _raw_clip(1, [A], ok, norm_type=float("-inf")) == nsg.DMUON_ERR_UNSUPPORTED
    # 4 x 8 bf16 = 64 bytes: the second gradient starts inside the first
    assert _raw_clip(2, [A, A + 32], ok * 2) == nsg.DMUON_ERR_INVALID_ARG
    assert "overlap" in nsg.dmuon_get_last_error()


def test_step_clipped_validation_errors():
    lib = nsg.library()
    A = 1 << 40
    vp = ctypes.c_void_p

    def call(max_norm, norm_type, shapes=((4, 8, 1),)):
        pa, ga, ba = (vp * 1)(A), (vp * 1)(A + 4096), (vp * 1)(A + 8192)
        return lib.dmuon_step_clipped(pa, ga, ba, nsg._shape_array(list(shapes)), 1, 0.02, 0.95, 1, 5,
                                      None, 0.0, max_norm, norm_type, None, None)
    assert call(float("inf"), 2.0) == nsg.DMUON_ERR_INVALID_ARG
    assert call(-0.5, 2.0) == nsg.DMUON_ERR_INVALID_ARG
    assert call(1.0, 0.5) == nsg.DMUON_ERR_UNSUPPORTED
    assert call(1.0, 2.0, ((4, 8, 9),)) == nsg.DMUON_ERR_INVALID_ARG


@pytest.mark.parametrize("seed", range(12))
def test_workspace_stays_under_the_cap(seed, monkeypatch):
    # random shape sets: the planned workspace fits the cap unless one matrix
    # alone needs more (that matrix then runs as a chunk of its own), and more
    # iterations never mean fewer launches
    rng = random.Random(100 + seed)
    cap_mb = rng.choice([64, 256, 1024, 8192])
    monkeypatch.setenv("DMUON_WS_CAP_MB", str(cap_mb))
    shapes = [(rng.choice([32, 256, 1000, 1408, 2048, 4096]), rng.choice([64, 512, 2816, 4096, 11008]),
               rng.randint(0, 1)) for _ in range(rng.randint(1, 40))]
    ws = nsg.dmuon_workspace_bytes(shapes, 5)
    single = max(nsg.dmuon_workspace_bytes([s], 5) for s in shapes)
    assert 0 < ws <= max(cap_mb << 20, single)
    assert nsg.dmuon_step_launches(shapes, 6) >= nsg.dmuon_step_launches(shapes, 5) >= nsg.dmuon_step_launches(shapes, 1)


def test_overlap_only_when_both_buffers_fit_the_cap(monkeypatch):
    # small layer: its largest matrix needs about 21 MB of workspace.  Under a
    # 20 MB cap two overlapped buffers would exceed the cap, so the plan runs
    # serially in one buffer; under 64 MB it overlaps with two buffers
    w = workloads.get("small_layer_bf16")
    shapes = [(r, c, 1) for r, c in w.shapes]

    def plan(cap, overlap):
        monkeypatch.setenv("DMUON_WS_CAP_MB", str(cap))
        monkeypatch.setenv("DMUON_OVERLAP", overlap)
        return nsg.dmuon_workspace_bytes(shapes, 5), nsg.dmuon_step_launches(shapes, 5)

    assert plan(20, "1") == plan(20, "0")
    ws_over, launches_over = plan(64, "1")
    ws_serial, launches_serial = plan(64, "0")
    assert ws_over <= 64 << 20 and launches_over > launches_serial


def _raw_buckets(count, ptrs, shapes, bucket_of, nb, max_norms, norm_types):
    lib = nsg._lib
    arr = (ctypes.c_void_p * max(1, count))(*ptrs)
    bo = (ctypes.c_int32 * max(1, count))(*bucket_of)
    mx = (ctypes.c_float * max(1, nb))(*max_norms)
    nt = (ctypes.c_float * max(1, nb))(*norm_types)
    return lib.dmuon_clip_grad_norm_buckets(arr, nsg._shape_array(shapes), count, bo, nb, mx, nt, None, None)


def test_clip_buckets_validation_errors():
    # every argument check comes before any device work, so this runs on the CPU
    A, B = 1 << 20, 1 << 21
    ok = [(4, 8, 1), (2, 2, 0)]
    E = nsg.DMUON_ERR_INVALID_ARG
    assert _raw_buckets(2, [A, B], ok, [0, 1], 0, [], []) == E                        # no bucket
    assert _raw_buckets(2, [A, B], ok, [0, 1], 129, [1.0] * 129, [2.0] * 129) == E    # too many
    assert _raw_buckets(2, [A, B], ok, [0, 2], 2, [1.0, 1.0], [2.0, 2.0]) == E        # index out of range
    assert _raw_buckets(2, [A, B], ok, [0, -1], 2, [1.0, 1.0], [2.0, 2.0]) == E
    assert _raw_buckets(2, [A, B], ok, [0, 1], 2, [1.0, float("nan")], [2.0, 2.0]) == E
    assert _raw_buckets(2, [A, B], ok, [0, 1], 2, [1.0, -1.0], [2.0, 2.0]) == E
    assert _raw_buckets(2, [A, B], ok, [0, 1], 2, [1.0, 1.0], [2.0, 3.0]) == nsg.DMUON_ERR_UNSUPPORTED
    assert _raw_buckets(2, [A, A + 16], ok, [0, 1], 2, [1.0, 1.0], [2.0, 2.0]) == E   # overlap across buckets
    assert _raw_buckets(2, [A, 0], ok, [0, 1], 2, [1.0, 1.0], [2.0, 2.0]) == E
    assert _raw_buckets(-1, [A], ok[:1], [0], 1, [1.0], [2.0]) == E


def test_clip_buckets_binding_flat_shapes():
    import torch
    f = nsg._flat_shape
    assert f(torch.empty(5, 6, 7)) == (30, 7)
    assert f(torch.empty(4096)) == (1, 4096)
    assert f(torch.empty(3 << 20)) == (3, 1 << 20)         # a long vector, split exactly
    r, c = f(torch.empty(2 ** 21 + 2))
    assert r * c == 2 ** 21 + 2 and max(r, c) <= 1 << 20
