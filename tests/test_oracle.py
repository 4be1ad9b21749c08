"""Pins for the fp64 oracle, against what the mathematics and the pages fix.

None of these re-types the oracle's own formula: the Newton-Schulz result is
checked against the SVD closed form (LAPACK), against invariances, against a
scalar map iterated by hand and against hand-computed recurrences.  The last
block plants plausible mistakes in copies of the oracle and checks that the
pins catch each of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import muon as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
A, B, C = om.DEFAULT_COEFFS


def scalar_poly(s, coeffs, steps):
    """Iterate f(s) = a s + b s^3 + c s^5 on singular values."""
    s = np.asarray(s, dtype=np.float64)
    for a, b, c in om.coeff_schedule(steps, coeffs):
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def ns_closed_form(m, steps, coeffs=None, eps=om.NORM_EPS):
    """U diag(f^k(sigma / (||M|| + eps))) V^T from LAPACK's SVD."""
    m = np.asarray(m, dtype=np.float64)
    u, s, vt = np.linalg.svd(m, full_matrices=False)
    fro = math.sqrt(float(np.sum(s * s)))
    return (u * scalar_poly(s / (fro + eps), coeffs, steps)) @ vt


def rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def gauss(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# --------------------------------------------------------------- golden pages
def test_defaults_match_pages():
    with open(os.path.join(GOLDEN, "hyperparameters.json")) as f:
        hp = json.load(f)
    import inspect
    sig = inspect.signature(om.muon_step)
    assert sig.parameters["lr"].default == hp["lr"]["value"]
    assert sig.parameters["momentum"].default == hp["momentum"]["value"]
    assert sig.parameters["ns_steps"].default == hp["ns_steps"]["value"]
    assert sig.parameters["nesterov"].default is hp["nesterov"]["value"]
    assert sig.parameters["wd"].default == hp["weight_decay"]["value"]
    assert om.LR_SHAPE_FACTOR == hp["lr_shape_factor"]["value"]


# ---------------------------------------------------------- closed form (SVD)
@pytest.mark.parametrize("shape", [(256, 512), (64, 48), (3, 7), (40, 40), (130, 33)])
def test_ns_matches_svd_closed_form(shape):
    m = gauss(shape, 11 + shape[0])
    o = om.newton_schulz(m, 5)
    assert o.shape == m.shape
    assert rel(o, ns_closed_form(m, 5)) < 1e-12


@pytest.mark.parametrize("coeffs", [(1.5, -0.5, 0.0), (15 / 8, -10 / 8, 3 / 8),
                                    [(3.0, -3.2, 1.2), (2.0, -1.5, 0.5), (1.5, -0.5, 0.0)]])
def test_ns_closed_form_custom_coeffs(coeffs):
    m = gauss((48, 80), 5)
    steps = 3
    assert rel(om.newton_schulz(m, steps, coeffs), ns_closed_form(m, steps, coeffs)) < 1e-12


def test_scalar_pin_rank_one():
    # 1 x n input: O = f^5(s) v/||v|| with s = ||v||/(||v||+eps); with eps=0, s=1.
    v = gauss((1, 257), 3)
    o = om.newton_schulz(v, 5, eps=0.0)
    f5 = 0.6964364094697522  # f^5(1) for (3.4445, -4.7750, 2.0315), iterated by hand
    assert np.allclose(o, f5 * v / np.linalg.norm(v), rtol=0, atol=1e-14)


def test_singular_value_band_default_coeffs():
    # For normalised sigma >= 1e-2 the 5-step default map stays in [0.6818, 1.1344];
    # on (0, 1] it never exceeds 1.2024.  Read the oracle's output along the input's
    # singular vectors: diag(U^T O V) are the output singular values.
    m = gauss((128, 300), 21)
    x = om.frobenius_normalize(m)
    u, s_in, vt = np.linalg.svd(x, full_matrices=False)
    out = np.diag(u.T @ om.newton_schulz(m, 5) @ vt.T)
    sel = s_in >= 1e-2
    assert sel.sum() > 100
    assert out[sel].min() >= 0.6818 and out[sel].max() <= 1.1344
    assert out.max() <= 1.2024 and out.min() > 0.0


@pytest.mark.parametrize("coeffs,steps", [((1.5, -0.5, 0.0), 25), ((15 / 8, -10 / 8, 3 / 8), 14)])
def test_convergent_polynomials_reach_polar_factor(coeffs, steps):
    m = gauss((64, 128), 8)
    u, _, vt = np.linalg.svd(m, full_matrices=False)
    assert rel(om.newton_schulz(m, steps, coeffs), u @ vt) < 1e-10


def test_default_quintic_does_not_converge_to_polar():
    # The default quintic oscillates inside its band rather than converging.
    m = gauss((64, 128), 8)
    u, _, vt = np.linalg.svd(m, full_matrices=False)
    assert rel(om.newton_schulz(m, 40), u @ vt) > 0.05


def test_diagonal_input():
    d = np.array([3.0, -1.0, 0.5, 2.0])
    m = np.diag(d)
    o = om.newton_schulz(m, 5, eps=0.0)
    s = np.abs(d) / np.linalg.norm(d)
    want = np.diag(np.sign(d) * scalar_poly(s, None, 5))
    assert np.allclose(o, want, atol=1e-14)


def test_tiny_2x3_brute_force():
    m = np.array([[1.0, 2.0, -1.0], [0.5, -0.25, 3.0]])
    # explicit loops for G = X X^T and the polynomial product
    x = m / (math.sqrt(sum(v * v for v in m.ravel())) + om.NORM_EPS)
    for _ in range(5):
        g = [[sum(x[i, k] * x[j, k] for k in range(3)) for j in range(2)] for i in range(2)]
        gg = [[sum(g[i][k] * g[k][j] for k in range(2)) for j in range(2)] for i in range(2)]
        p = [[B * g[i][j] + C * gg[i][j] for j in range(2)] for i in range(2)]
        x = np.array([[A * x[i, j] + sum(p[i][k] * x[k, j] for k in range(2))
                       for j in range(3)] for i in range(2)])
    assert np.allclose(om.newton_schulz(m, 5), x, atol=1e-14)


# ------------------------------------------------------------- invariances
def test_transpose_equivariance():
    m = gauss((70, 150), 4)
    assert np.allclose(om.newton_schulz(m.T, 5), om.newton_schulz(m, 5).T, atol=1e-13)


@pytest.mark.parametrize("c", [1e-2 / 100.0, 7.5, 1e3])
def test_scale_invariance(c):
    m = gauss((50, 90), 6)
    m = m / np.linalg.norm(m)
    # exact with eps=0; with eps, within eps/||cM||
    assert np.allclose(om.newton_schulz(c * m, 5, eps=0.0), om.newton_schulz(m, 5, eps=0.0),
                       atol=1e-12)
    if c * 1.0 >= 1e-2:
        assert rel(om.newton_schulz(c * m, 5), om.newton_schulz(m, 5)) < 1e-5


def test_zero_matrix_gives_zero_update():
    o = om.newton_schulz(np.zeros((8, 16)), 5)
    assert np.all(o == 0.0)


def test_zero_steps_is_normalised_input():
    m = gauss((10, 20), 2)
    o = om.newton_schulz(m, 0)
    assert abs(np.linalg.norm(o) - np.linalg.norm(m) / (np.linalg.norm(m) + om.NORM_EPS)) < 1e-14
    assert np.allclose(o * (np.linalg.norm(m) + om.NORM_EPS), m, atol=1e-13)


# ---------------------------------------------------------------- momentum
def test_momentum_hand_computed_2x2():
    buf0 = np.array([[1.0, -2.0], [0.5, 0.0]])
    g = np.array([[0.1, 0.2], [-0.3, 1.0]])
    b1, x1 = om.momentum_update(buf0, g, 0.5, True)
    assert np.allclose(b1, [[0.6, -0.8], [-0.05, 1.0]], atol=1e-15)
    assert np.allclose(x1, [[0.4, -0.2], [-0.325, 1.5]], atol=1e-15)
    b2, x2 = om.momentum_update(b1, np.zeros((2, 2)), 0.5, True)
    assert np.allclose(b2, [[0.3, -0.4], [-0.025, 0.5]], atol=1e-15)
    assert np.allclose(x2, [[0.15, -0.2], [-0.0125, 0.25]], atol=1e-15)
    b3, x3 = om.momentum_update(b1, g, 0.5, False)
    assert np.allclose(x3, b3) and np.allclose(b3, [[0.4, -0.2], [-0.325, 1.5]], atol=1e-15)


def test_momentum_constant_gradient_closed_form():
    mu, t = 0.95, 7
    g = gauss((3, 4), 9)
    buf = np.zeros_like(g)
    for _ in range(t):
        buf, _ = om.momentum_update(buf, g, mu, True)
    assert np.allclose(buf, g * (1 - mu ** t) / (1 - mu), atol=1e-13)


def test_single_matrix_zero_buffer_special_case():
    # zero buffer: x0 = (1 + mu) g, so O = NS(g) up to eps; lr_eff = 0.02*0.2*sqrt(512)
    p = gauss((256, 512), 1, 0.02)
    g = gauss((256, 512), 2)
    ps, bs, os_ = om.muon_step([p], [g], [np.zeros_like(g)])
    assert np.allclose(bs[0], g)
    assert rel(os_[0], om.newton_schulz(g, 5)) < 1e-9
    assert abs(0.02 * om.lr_scale(256, 512) - 0.0905097) < 1e-7
    assert np.allclose(ps[0], p - 0.02 * 0.2 * math.sqrt(512) * os_[0], atol=1e-15)


# ------------------------------------------------------------------ update
def test_update_hand_computed():
    p = np.array([[1.0, 2.0, 3.0]])
    o = np.array([[0.5, -0.5, 1.0]])
    s = 0.1 * 0.2 * math.sqrt(3.0)
    want = np.array([[0.95 - 0.5 * s, 1.9 + 0.5 * s, 2.85 - s]])
    assert np.allclose(om.apply_update(p, o, 0.1, 0.5), want, atol=1e-15)


def test_update_tall_uses_max_dimension():
    p = np.zeros((9, 4))
    o = np.ones((9, 4))
    assert np.allclose(om.apply_update(p, o, 1.0, 0.0), -0.2 * 3.0)


# ------------------------------------------------------------------ groups
def test_shape_groups_hand_computed():
    shapes = [(4, 8, 1), (2, 2, 1), (4, 8, 1), (4, 8, 0), (2, 2, 1), (8, 4, 1)]
    g, order, n = om.shape_groups(shapes)
    assert g == [0, 1, 0, 2, 1, 3]
    assert order == [0, 2, 1, 4, 3, 5]
    assert n == 4
    assert om.shape_groups([]) == ([], [], 0)


def test_shape_groups_brute_force_properties():
    rng = np.random.default_rng(0)
    for trial in range(50):
        cnt = int(rng.integers(1, 40))
        shapes = [(int(rng.integers(1, 4)), int(rng.integers(1, 4)), int(rng.integers(0, 2)))
                  for _ in range(cnt)]
        g, order, n = om.shape_groups(shapes)
        assert sorted(order) == list(range(cnt))
        # same key <=> same group
        for i in range(cnt):
            for j in range(cnt):
                assert (g[i] == g[j]) == (shapes[i] == shapes[j])
        # first appearance order of group ids
        firsts = [g.index(k) for k in range(n)]
        assert firsts == sorted(firsts)
        # order is grouped, ascending inside a group
        pos = 0
        for k in range(n):
            mem = [i for i in range(cnt) if g[i] == k]
            assert order[pos:pos + len(mem)] == mem
            pos += len(mem)


# --------------------------------------------------------- planted mistakes
def _mutant_dropped_c(x, steps, coeffs=None):
    for a, b, c in om.coeff_schedule(steps, coeffs):
        g = x @ x.T
        x = a * x + (b * g) @ x
    return x


def _mutant_sign_b(x, steps, coeffs=None):
    for a, b, c in om.coeff_schedule(steps, coeffs):
        g = x @ x.T
        x = a * x + (-b * g + c * (g @ g)) @ x
    return x


def _mutant_wrong_gram(x, steps, coeffs=None):
    for a, b, c in om.coeff_schedule(steps, coeffs):
        g = x.T @ x          # Gram over the larger side, applied from the right
        x = a * x + x @ (b * g + c * (g @ g))
        x = x * 1.0001
    return x


def _mutant_transposed_apply(x, steps, coeffs=None):
    for a, b, c in om.coeff_schedule(steps, coeffs):
        g = x @ x.T
        p = b * g + c * (g @ g)
        p = p + np.triu(np.ones_like(p), 1) * 1e-3   # breaks the symmetry p(G) has
        x = a * x + p.T @ x
    return x


@pytest.mark.parametrize("mutant", [_mutant_dropped_c, _mutant_sign_b, _mutant_wrong_gram,
                                    _mutant_transposed_apply])
def test_pins_catch_planted_iteration_mistakes(monkeypatch, mutant):
    m = gauss((40, 72), 13)
    monkeypatch.setattr(om, "gram_ns_iterations", mutant)
    assert rel(om.newton_schulz(m, 5), ns_closed_form(m, 5)) > 1e-6


def test_orientation_runs_over_smaller_side():
    x, t = om.orient(gauss((90, 30), 3))
    assert t is True and x.shape == (30, 90)
    x, t = om.orient(gauss((30, 30), 3))
    assert t is False and x.shape == (30, 30)


def test_pins_catch_planted_momentum_mistakes(monkeypatch):
    buf0 = np.array([[1.0, -2.0], [0.5, 0.0]])
    g = np.array([[0.1, 0.2], [-0.3, 1.0]])

    def old_buffer_nesterov(buf, g, mu, nesterov):
        nb = mu * buf + g
        return nb, g + mu * buf

    def lerp_buffer(buf, g, mu, nesterov):
        nb = mu * buf + (1 - mu) * g
        return nb, g + mu * nb

    for mut in (old_buffer_nesterov, lerp_buffer):
        b1, x1 = mut(buf0, g, 0.5, True)
        ok = np.allclose(b1, [[0.6, -0.8], [-0.05, 1.0]]) and \
            np.allclose(x1, [[0.4, -0.2], [-0.325, 1.5]])
        assert not ok


def test_pins_catch_planted_update_mistakes():
    p = np.array([[1.0, 2.0, 3.0]])
    o = np.array([[0.5, -0.5, 1.0]])
    s = 0.1 * 0.2 * math.sqrt(3.0)
    want = np.array([[0.95 - 0.5 * s, 1.9 + 0.5 * s, 2.85 - s]])
    wrong = [p * (1 - 0.1 * 0.5) - 0.1 * 0.2 * math.sqrt(1.0) * o,          # min dim
             p * (1 - 0.1 * s * 0.5) - 0.1 * s * o,                           # scaled decay
             p - 0.1 * s * o]                                                 # no decay
    for w in wrong:
        assert not np.allclose(w, want, atol=1e-12)



# ---------------------------------------------------------------- clipping
def test_clip_hand_computed_l2():
    g1 = np.array([[3.0, 4.0]])
    g2 = np.array([[0.0, 12.0]])
    out, total, coef = om.clip_grad_norm([g1, g2], 6.5)
    assert total == 13.0
    assert abs(coef - 6.5 / (13.0 + 1e-6)) < 1e-15
    assert np.allclose(out[0], g1 * 6.5 / (13.0 + 1e-6)) and np.allclose(out[1], g2 * coef)


def test_clip_below_threshold_is_identity():
    g = gauss((3, 5), 1)
    out, total, coef = om.clip_grad_norm([g], 1e6)
    assert coef == 1.0 and np.array_equal(out[0], g)
    assert abs(total - np.linalg.norm(g)) < 1e-12


def test_clip_inf_and_l1_norms():
    g1 = np.array([[1.0, -7.0]])
    g2 = np.array([[2.0, 0.5], [-3.0, 0.0]])
    _, t_inf, c_inf = om.clip_grad_norm([g1, g2], 3.5, float("inf"))
    assert t_inf == 7.0 and abs(c_inf - 3.5 / (7.0 + 1e-6)) < 1e-15
    _, t_1, _ = om.clip_grad_norm([g1, g2], 1.0, 1.0)
    assert t_1 == 1.0 + 7.0 + 2.0 + 0.5 + 3.0


def test_clip_global_norm_couples_matrices():
    # the clip is global: a large gradient also shrinks a small one
    small, big = np.full((2, 2), 1e-3), np.full((2, 2), 100.0)
    out, total, coef = om.clip_grad_norm([small, big], 1.0)
    assert abs(total - np.sqrt(4 * 1e-6 + 4 * 1e4)) < 1e-9
    assert np.allclose(out[0], small * coef) and coef < 0.01


@pytest.mark.parametrize("norm_type", [1.0, 2.0, float("inf")])
@pytest.mark.parametrize("where", [0, 1, 2])
def test_clip_nan_anywhere_gives_nan_total(norm_type, where):
    # PyTorch's clip_grad_norm_ (whose name and max_norm argument the clipping
    # section gives DMuon's clip) reduces with sum / max, both of which keep a
    # NaN wherever it sits, and its clamp keeps the NaN coefficient: every
    # gradient becomes NaN
    gs = [gauss((3, 4), 20 + k) for k in range(3)]
    gs[where][1, 2] = np.nan
    out, total, coef = om.clip_grad_norm(gs, 1.0, norm_type)
    assert np.isnan(total) and np.isnan(coef)
    assert all(np.isnan(a).all() for a in out)


@pytest.mark.parametrize("norm_type", [1.0, 2.0, float("inf")], ids=["l1", "l2", "linf"])
@pytest.mark.parametrize("case", ["clipped", "below", "nan", "inf", "zero"])
def test_clip_matches_pytorch_clip_grad_norm(norm_type, case):
    # the reading is PyTorch's formula: its own routine (CPU, fp64) pins the
    # total, the coefficient and the clipped values, non-finite cases included
    gs = [gauss((5, 7), 40), gauss((3, 11), 41) * 3.0, gauss((1, 4), 42)]
    max_norm = 2.5 if case != "below" else 1e6
    if case == "nan":
        gs[1][2, 3] = np.nan
    elif case == "inf":
        gs[2][0, 1] = -np.inf
    elif case == "zero":
        gs = [np.zeros_like(g) for g in gs]
    ts = [torch.nn.Parameter(torch.zeros(g.shape, dtype=torch.float64)) for g in gs]
    for t, g in zip(ts, gs):
        t.grad = torch.from_numpy(g.copy())
    want_total = float(torch.nn.utils.clip_grad_norm_(ts, max_norm, norm_type=norm_type))
    out, total, coef = om.clip_grad_norm(gs, max_norm, norm_type)
    assert (np.isnan(total) and np.isnan(want_total)) or total == pytest.approx(want_total, rel=1e-12, abs=0)
    for o, t in zip(out, ts):
        w = t.grad.numpy()
        assert np.array_equal(np.isnan(o), np.isnan(w))
        ok = ~np.isnan(w)
        assert np.allclose(o[ok], w[ok], rtol=1e-12, atol=0)


def test_clip_infinity_gives_zero_coefficient():
    gs = [np.array([[1.0, np.inf]]), np.array([[2.0]])]
    for norm_type in (1.0, 2.0, float("inf")):
        out, total, coef = om.clip_grad_norm(gs, 1.0, norm_type)
        assert total == np.inf and coef == 0.0
        assert np.isnan(out[0][0, 1]) and out[0][0, 0] == 0.0 and out[1][0, 0] == 0.0


def test_clip_buckets_match_pytorch_per_bucket():
    # Training Guide, "Fused CUDA clip for regular / Muon / AdamW": every bucket
    # keeps the semantics of its own clip.  PyTorch's clip_grad_norm_, called
    # once per bucket (CPU, fp64), pins totals, coefficients and values; the
    # buckets differ in norm type, max_norm, size, and one holds a NaN (which
    # must not reach the others) and one is below its bound
    buckets = [[gauss((5, 7), 50), gauss((2, 9), 51) * 4.0],
               [gauss((3, 3), 52)],
               [gauss((1, 13), 53) * 0.01, gauss((6, 2), 54)],
               [gauss((4, 4), 55)]]
    buckets[3][0][1, 2] = np.nan
    max_norms = [1.5, 0.25, 1e6, 1.0]
    norm_types = [2.0, float("inf"), 1.0, 2.0]
    got = om.clip_grad_norm_buckets(buckets, max_norms, norm_types)
    assert len(got) == 4
    for bucket, mx, nt, (out, total, coef) in zip(buckets, max_norms, norm_types, got):
        ts = [torch.nn.Parameter(torch.zeros(g.shape, dtype=torch.float64)) for g in bucket]
        for t, g in zip(ts, bucket):
            t.grad = torch.from_numpy(g.copy())
        want = float(torch.nn.utils.clip_grad_norm_(ts, mx, norm_type=nt))
        assert (np.isnan(total) and np.isnan(want)) or total == pytest.approx(want, rel=1e-12, abs=0)
        for o, t in zip(out, ts):
            w = t.grad.numpy()
            assert np.array_equal(np.isnan(o), np.isnan(w))
            assert np.allclose(o[~np.isnan(w)], w[~np.isnan(w)], rtol=1e-12, atol=0)
    # the NaN stayed in its bucket; the bucket below its bound is unchanged
    assert not any(np.isnan(o).any() for _, (out, _, _) in zip(range(3), got) for o in out)
    assert got[2][2] == 1.0 and all(np.array_equal(o, g) for o, g in zip(got[2][0], buckets[2]))


def test_clip_buckets_empty_bucket_and_argument_errors():
    out, total, coef = om.clip_grad_norm_buckets([[], [gauss((2, 2), 56)]], [1.0, 1.0], [2.0, 2.0])[0]
    assert out == [] and total == 0.0 and coef == 1.0
    with pytest.raises(ValueError):
        om.clip_grad_norm_buckets([[gauss((2, 2), 57)]], [1.0, 2.0], [2.0])
