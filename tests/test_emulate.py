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


def test_momentum_fp32_without_nesterov_hand_values():
    # x0 is the new buffer itself; bf16 storage rounds both the same way:
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 (to even: 1), 1 + 3 * 2^-8 a tie
    # between 1 + 2^-7 and 1 + 2^-6 (to even: 1 + 2^-6)
    buf = np.array([[1.0, -2.0, 1.0, 1.0]], dtype=np.float32)
    g = np.array([[0.5, 0.25, 2.0 ** -8, 3 * 2.0 ** -8]], dtype=np.float32)
    nb, x0 = em.momentum_fp32(buf, g, 0.5, False, "f32")
    assert np.array_equal(nb, np.array([[1.0, -0.75, 0.5 + 2.0 ** -8, 0.5 + 3 * 2.0 ** -8]], dtype=np.float32))
    assert np.array_equal(x0, nb)
    nb, x0 = em.momentum_fp32(buf, g, 1.0, False, "bf16")
    assert np.array_equal(nb, np.array([[1.5, -1.75, 1.0, 1.0 + 2.0 ** -6]], dtype=np.float32))
    assert np.array_equal(x0, nb)


def test_update_fp32_with_weight_decay_hand_values():
    # 1 x 100: sqrt(max(rows, cols)) = 10, so with lr = 0.25 the step scale is
    # 0.25 * 0.2 * 10 = 0.5 and the decay (unscaled lr) 1 - 0.25 * 2 = 0.5; a
    # decay taken with the scaled lr would be 0
    p = np.zeros((1, 100), dtype=np.float32)
    o = np.zeros((1, 100), dtype=np.float32)
    p[0, :4] = [3.0, -1.0, 1.0, 1.0]
    o[0, :4] = [1.0, 2.0, -(2.0 ** -8), -3 * 2.0 ** -8]
    out = em.update_fp32(p, o, 0.25, 2.0, "f32")
    assert np.array_equal(out[0, :4], np.array([1.0, -1.5, 0.5 + 2.0 ** -9, 0.5 + 3 * 2.0 ** -9], dtype=np.float32))
    assert not out[0, 4:].any()
    # bf16: 0.5 + 2^-9 is a tie (to even: 0.5); 0.5 + 3 * 2^-9 a tie (to 0.5 + 2^-7)
    out = em.update_fp32(p, o, 0.25, 2.0, "bf16")
    assert np.array_equal(out[0, :4], np.array([1.0, -1.5, 0.5, 0.5 + 2.0 ** -7], dtype=np.float32))


def test_clip_scale_fp32_hand_values():
    g = np.array([[2.0, -6.0, 0.5]], dtype=np.float32)
    assert np.array_equal(em.clip_scale_fp32(g, 0.25, "f32"), np.array([[0.5, -1.5, 0.125]], dtype=np.float32))
    # one fp32 product, then bf16 storage: 1 * (1 + 2^-8) is a tie (to 1);
    # 3 * (1 + 2^-8) = 3.01171875 lies above the midpoint 3.0078125 (to 3.015625)
    g = np.array([[1.0, 3.0]], dtype=np.float32)
    assert np.array_equal(em.clip_scale_fp32(g, 1.0 + 2.0 ** -8, "bf16"), np.array([[1.0, 3.015625]], dtype=np.float32))
    # the coefficient is rounded to fp32 once: 1/3 -> 0x3EAAAAAB, and 2^24 times
    # it is exactly 5592405.5
    g = np.array([[2.0 ** 24]], dtype=np.float32)
    assert em.clip_scale_fp32(g, 1.0 / 3.0, "f32")[0, 0] == np.float32(5592405.5)
    # coefficient 0 turns an infinity into NaN; a NaN coefficient makes every value NaN
    out = em.clip_scale_fp32(np.array([[np.inf, 1.0]], dtype=np.float32), 0.0, "f32")
    assert np.isnan(out[0, 0]) and out[0, 1] == 0.0
    assert np.isnan(em.clip_scale_fp32(np.array([[1.0, 0.0]], dtype=np.float32), float("nan"), "bf16")).all()
