"""Pins for the fp32 rounding-contract emulation used by the bit-exact tests."""
import numpy as np
import torch

from oracle import emulate as em


def test_bf16_round_matches_torch_conversion():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 100000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0, 3.3895314e38,
                                  1e-40, -1e-40], dtype=np.float32)]).astype(np.float32)
    # exact ties: low half == 0x8000
    u = rng.integers(0, 2**32, 1000, dtype=np.uint64).astype(np.uint32)
    u = (u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    x = np.concatenate([x, u.view(np.float32)])
    x = x[np.isfinite(x)]
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    got = em.bf16_round(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_momentum_fp32_hand_values():
    buf = np.array([[1.0, -2.0]], dtype=np.float32)
    g = np.array([[0.5, 0.25]], dtype=np.float32)
    nb, x0 = em.momentum_fp32(buf, g, 0.5, True, "f32")
    assert np.array_equal(nb, np.array([[1.0, -0.75]], dtype=np.float32))
    assert np.array_equal(x0, np.array([[1.0, -0.125]], dtype=np.float32))


def test_update_fp32_hand_values():
    p = np.array([[1.0, 2.0]], dtype=np.float32)
    o = np.array([[1.0, -1.0]], dtype=np.float32)
    out = em.update_fp32(p, o, 0.5, 0.0, "f32")
    s = np.float32(0.5 * 0.2 * np.sqrt(2.0))
    assert np.array_equal(out, np.array([[np.float32(1.0) - s, np.float32(2.0) + s]], dtype=np.float32))
