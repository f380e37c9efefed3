"""Pins for the fp64 oracle: closed forms, invariants, library routines, brute
force and values printed on the pages.  None of these re-types the oracle's
own formula; each is chosen so that a plausible slip in the oracle (a dropped
term, a sign, a transposed operand, a wrong coefficient) fails at least one.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle as orc
from matrix_orthogonalising_optimizer_02_b200 import workloads

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_values.json")))


def _orth(r, n, k):
    q, _ = np.linalg.qr(r.standard_normal((n, k)))
    return q


def _svd_polynomial_ns(X0, schedule, eps=1e-7):
    """Closed form: NS acts on each singular value by the scalar polynomial
    phi_t(s) = a s + b s^3 + c s^5 and leaves the singular vectors alone."""
    X = np.asarray(X0, np.float64)
    U, s, Vt = np.linalg.svd(X / (np.linalg.norm(X) + eps), full_matrices=False)
    for (a, b, c) in schedule:
        s = a * s + b * s ** 3 + c * s ** 5
    return (U * s) @ Vt


# --------------------------------------------------------------------- rounding

def test_bf16_rounding_matches_torch():
    r = workloads.rng(5)
    x = np.concatenate([
        r.standard_normal(20000) * 10.0 ** r.integers(-30, 30, 20000),
        np.array([0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, 3.0e38, 1e-40]),
        # exact ties between two bf16 neighbours (round to even either way)
        (np.arange(1, 200, dtype=np.float64) * 2 ** -8 + 2 ** -9) * 4.0,
    ])
    ours = orc.round_to_bf16(x)
    ref = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)
    assert np.isnan(orc.round_to_bf16(np.array([np.nan])))[0]


def test_f32_rounding_is_ieee():
    x = np.array([1.0 + 2.0 ** -30, 0.1, -7.25, 1e-50])
    assert np.array_equal(orc.round_to_f32(x), x.astype(np.float32).astype(np.float64))


# --------------------------------------------------------------------- coefficients

def test_coefficients_are_the_printed_ones():
    assert tuple(orc.KJ_COEFFS) == tuple(GOLDEN["kj_coeffs"]["value"])
    assert tuple(orc.TEXTBOOK_COEFFS) == tuple(GOLDEN["textbook_coeffs"]["value"])
    assert orc.NS_EPS == GOLDEN["ns_eps"]["value"]
    num = GOLDEN["taylor_numerators"]
    assert np.allclose(np.array(num["value"]) / num["denominator"], orc.TEXTBOOK_COEFFS, rtol=0, atol=0)


def test_textbook_is_second_order_taylor_of_inverse_sqrt():
    # Taylor coefficients of f(t) = t^(-1/2) at t = 1 from central differences
    f = lambda t: t ** -0.5
    h = 1e-3
    f0, f1 = f(1.0), (f(1 + h) - f(1 - h)) / (2 * h)
    f2 = (f(1 + h) - 2 * f(1.0) + f(1 - h)) / h ** 2
    # f0 + f1 (t-1) + f2/2 (t-1)^2 expanded in powers of t
    poly = np.array([f0 - f1 + f2 / 2, f1 - f2, f2 / 2])
    assert np.allclose(poly, orc.TEXTBOOK_COEFFS, atol=1e-5)
    a, b, c = orc.TEXTBOOK_COEFFS
    assert a + b + c == 1.0                       # phi(1) = 1
    assert a + 3 * b + 5 * c == 0.0               # phi'(1) = 0


def test_schedules():
    assert orc.fixed_schedule(5) == [orc.KJ_COEFFS] * 5
    hy = orc.hybrid_schedule()
    g = GOLDEN["hybrid_schedule"]
    assert hy[: g["n_fast"]] == [orc.KJ_COEFFS] * g["n_fast"]
    assert hy[g["n_fast"]:] == [orc.TEXTBOOK_COEFFS] * g["n_stable"]


# --------------------------------------------------------------------- msign

def test_msign_of_constructed_svd():
    r = workloads.rng(11)
    for (m, n) in [(7, 5), (5, 7), (6, 6), (40, 13)]:
        k = min(m, n)
        U, V = _orth(r, m, k), _orth(r, n, k)
        s = np.sort(r.uniform(0.1, 10.0, k))[::-1]
        M = (U * s) @ V.T
        assert np.allclose(orc.msign_svd(M), U @ V.T, atol=1e-12)


def test_msign_is_closest_orthogonal_brute_force():
    r = workloads.rng(12)
    for (m, n) in [(3, 3), (4, 2)]:
        M = r.standard_normal((m, n))
        O = orc.msign_svd(M)
        best = np.linalg.norm(M - O)
        k = min(m, n)
        for _ in range(10000):
            Q = _orth(r, m, k)
            if m == n and r.random() < 0.5:
                Q[:, 0] *= -1.0          # include reflections
            cand = Q if m >= n else Q.T
            assert best <= np.linalg.norm(M - cand) + 1e-12


def test_msign_equals_polar_inverse_sqrt_form():
    r = workloads.rng(13)
    M = r.standard_normal((9, 6))
    w, Q = np.linalg.eigh(M.T @ M)
    inv_sqrt = (Q / np.sqrt(w)) @ Q.T
    assert np.allclose(M @ inv_sqrt, orc.msign_svd(M), atol=1e-12)
    w2, Q2 = np.linalg.eigh(M @ M.T)
    # (M M^T)^(-1/2) M on the range of M (M M^T is singular here: use pinv)
    pinv_sqrt = (Q2[:, -6:] / np.sqrt(w2[-6:])) @ Q2[:, -6:].T
    assert np.allclose(pinv_sqrt @ M, orc.msign_svd(M), atol=1e-12)


# --------------------------------------------------------------------- Newton-Schulz

@pytest.mark.parametrize("shape", [(64, 48), (48, 64), (64, 64), (96, 40)])
@pytest.mark.parametrize("sched", ["kj5", "hybrid", "textbook3"])
def test_ns_is_polynomial_of_singular_values(shape, sched):
    schedule = {"kj5": orc.fixed_schedule(5), "hybrid": orc.hybrid_schedule(),
                "textbook3": orc.fixed_schedule(3, orc.TEXTBOOK_COEFFS)}[sched]
    r = workloads.rng(21)
    X0 = r.standard_normal(shape)
    got = orc.newton_schulz(X0, schedule)
    want = _svd_polynomial_ns(X0, schedule)
    assert np.linalg.norm(got - want) <= 1e-10 * np.linalg.norm(want)


def test_ns_rank_one_gives_phi_T_of_one():
    r = workloads.rng(22)
    u, v = _orth(r, 30, 1), _orth(r, 20, 1)
    M = 4.0 * (u @ v.T)
    s = 4.0 / (4.0 + orc.NS_EPS)
    a, b, c = orc.KJ_COEFFS
    for _ in range(5):
        s = a * s + b * s ** 3 + c * s ** 5
    assert np.allclose(orc.newton_schulz(M, orc.fixed_schedule(5)), s * (u @ v.T), atol=1e-12)
    # tall input goes through the transpose branch; same answer transposed
    assert np.allclose(orc.newton_schulz(M.T, orc.fixed_schedule(5)), s * (v @ u.T), atol=1e-12)


def test_ns_equivariance_and_transpose():
    r = workloads.rng(23)
    X = r.standard_normal((24, 40))
    Q, R = _orth(r, 24, 24), _orth(r, 40, 40)
    sch = orc.fixed_schedule(5)
    base = orc.newton_schulz(X, sch)
    assert np.allclose(orc.newton_schulz(Q @ X @ R, sch), Q @ base @ R, atol=1e-10)
    assert np.allclose(orc.newton_schulz(X.T, sch), base.T, atol=1e-12)


def test_ns_band_after_five_steps():
    lo, hi = GOLDEN["ns_band_after_5_steps"]["value"]
    r = workloads.rng(24)
    for (m, n) in [(64, 256), (256, 64), (128, 512), (100, 300)]:
        X = r.standard_normal((m, n))
        s = np.linalg.svd(orc.newton_schulz(X, orc.fixed_schedule(5)), compute_uv=False)
        assert s.min() >= lo and s.max() <= hi


def test_textbook_iteration_converges_to_msign():
    r = workloads.rng(25)
    U, V = _orth(r, 40, 30), _orth(r, 30, 30)
    M = (U * np.linspace(1.0, 3.0, 30)) @ V.T            # well conditioned
    got = orc.newton_schulz(M, orc.fixed_schedule(60, orc.TEXTBOOK_COEFFS))
    assert np.allclose(got, orc.msign_svd(M), atol=1e-12)
    hy = orc.newton_schulz(M, orc.hybrid_schedule())
    s = np.linalg.svd(hy, compute_uv=False)
    assert np.all(np.abs(s - 1.0) < 0.05)


def test_frobenius_prescale_bounds_spectral_norm():
    r = workloads.rng(26)
    for shape in [(10, 10), (5, 30), (30, 5)]:
        X = r.standard_normal(shape) * 100.0
        s = np.linalg.svd(orc.frobenius_prescale(X), compute_uv=False)
        assert s.max() <= 1.0
        assert s.max() >= 1.0 / np.sqrt(min(shape)) - 1e-12       # ||.||_F <= sqrt(r) ||.||_2
    D = np.diag([3.0, 4.0])
    assert np.allclose(orc.frobenius_prescale(D, eps=0.0), np.diag([0.6, 0.8]))


# --------------------------------------------------------------------- scale and update

def test_scale_modes_page_example():
    ex = GOLDEN["scale_example_1024x4096"]
    assert orc.scale_factor(ex["rows"], ex["cols"], "kellerjordan") == ex["kellerjordan"]
    assert np.isclose(orc.scale_factor(ex["rows"], ex["cols"], "moonlight"), ex["moonlight"], rtol=1e-15)
    assert orc.scale_factor(1024, 4096, "mup") == 0.5
    assert orc.scale_factor(4096, 1024, "kellerjordan") == 2.0
    assert orc.scale_factor(4096, 1024, "naive") == 1.0
    assert np.isclose(orc.scale_factor(256, 128, "moonlight"), 3.2)


def test_zero_gradient_gives_pure_decay():
    r = workloads.rng(31)
    W0 = orc.round_to_bf16(r.standard_normal((48, 80)) * 0.02)
    out = orc.muon_step(W0, np.zeros_like(W0), np.zeros_like(W0), lr=0.02, weight_decay=0.1)
    assert np.all(out["O"] == 0.0)
    assert np.array_equal(out["W1"], orc.round_to_bf16((1 - 0.02 * 0.1) * W0))


def test_update_decays_old_weights_then_steps():
    # decoupled decay multiplies the *old* W only; the step is not decayed
    r = workloads.rng(32)
    W0, O = r.standard_normal((6, 9)), r.standard_normal((6, 9))
    W1 = orc.muon_update(W0, O, lr=0.5, weight_decay=0.4, scale=2.0)
    assert np.allclose(orc.muon_update(W0, 0 * O, 0.5, 0.4, 2.0), 0.8 * W0)
    assert np.allclose(orc.muon_update(0 * W0, O, 0.5, 0.4, 2.0), -1.0 * O)
    assert np.allclose(W1, 0.8 * W0 - 1.0 * O)


def test_momentum_special_cases():
    r = workloads.rng(33)
    M0, G = r.standard_normal((5, 7)), r.standard_normal((5, 7))
    M1, g = orc.momentum(M0, G, beta=0.0)
    assert np.array_equal(M1, G) and np.array_equal(g, G)
    M1, g = orc.momentum(M0, 0 * G, beta=0.95)
    assert np.allclose(M1, 0.95 * M0) and np.array_equal(g, M1)
    # two steps from zero accumulate a geometric sum
    G2 = r.standard_normal((5, 7))
    M1, _ = orc.momentum(np.zeros_like(G), G, 0.9)
    M2, g2 = orc.momentum(M1, G2, 0.9, nesterov=True)
    assert np.allclose(M2, 0.9 * G + G2)
    assert np.allclose(g2, 0.9 * M2 + G2)


def test_muon_step_bf16_input_cast():
    r = workloads.rng(34)
    W, G = r.standard_normal((20, 12)) * 0.02, r.standard_normal((20, 12)) * 1e-3
    out = orc.muon_step(W, G, np.zeros_like(G), lr=0.02)
    assert np.array_equal(out["X0"], orc.round_to_bf16(G))
    out32 = orc.muon_step(W, G, np.zeros_like(G), lr=0.02, fp32_mode=True, w_dtype="f32")
    assert np.array_equal(out32["X0"], orc.round_to_f32(G))


# --------------------------------------------------------------------- Stiefel / Cayley

def test_tangent_projection_properties():
    r = workloads.rng(41)
    n, k = 50, 12
    W = _orth(r, n, k)
    G = r.standard_normal((n, k))
    V = orc.project_tangent(W, G)
    assert np.max(np.abs(V.T @ W + W.T @ V)) < 1e-12              # tangent condition
    assert np.allclose(orc.project_tangent(W, V), V, atol=1e-12)   # idempotent
    S = r.standard_normal((k, k)); S = S + S.T
    assert np.allclose(orc.project_tangent(W, W @ S), 0.0, atol=1e-12)   # normal space removed
    K = r.standard_normal((k, k)); K = K - K.T
    Z = r.standard_normal((n, k)); Z = Z - W @ (W.T @ Z)
    T = W @ K + Z                                                    # a tangent vector
    assert np.allclose(orc.project_tangent(W, T), T, atol=1e-12)


def test_cayley_two_by_one_is_a_rotation():
    # A = v J with J the 2x2 rotation generator: the Cayley factor is a
    # rotation and e1 maps to ((1 - t^2), -2t) / (1 + t^2), t = c v.
    for lr, v in [(0.01, 3.0), (0.5, -1.3), (2.0, 0.7)]:
        W = np.array([[1.0], [0.0]])
        V = np.array([[0.0], [v]])
        t = lr / 2 * v
        want = np.array([[1 - t * t], [-2 * t]]) / (1 + t * t)
        assert np.allclose(orc.cayley_dense(W, V, lr), want, atol=1e-14)
        assert np.allclose(orc.cayley_woodbury(W, V, lr), want, atol=1e-14)


def test_cayley_preserves_orthonormality_and_woodbury_matches_dense():
    r = workloads.rng(42)
    for (n, k, lr) in [(64, 16, 1e-2), (200, 30, 0.3), (128, 64, 1.0)]:
        W = _orth(r, n, k)
        V = orc.project_tangent(W, r.standard_normal((n, k)))
        Wd = orc.cayley_dense(W, V, lr)
        Ww = orc.cayley_woodbury(W, V, lr)
        assert orc.orthogonality_error(Wd) < 1e-12
        assert np.max(np.abs(Wd - Ww)) < 1e-12
        # the dense Cayley factor itself is orthogonal (skew A)
        c = lr / 2
        A = V @ W.T - W @ V.T
        Q = np.linalg.solve(np.eye(n) + c * A, np.eye(n) - c * A)
        assert np.max(np.abs(Q.T @ Q - np.eye(n))) < 1e-12


def test_cayley_doubled_resolvent_form_matches_woodbury():
    """(I + cA)^-1 (I - cA) = 2 (I + cA)^-1 - I, so with the rank-2k factorisation A = U B the
    retraction is W - 2 U C^-1 (c B W): the same map as the page's Woodbury steps (b, y = B b,
    z = C^-1 y, W_new = b - c U z) with y replaced by c B W = [cQ; -cP^T].  Written out here in
    fp64 from the factorisation and compared with the oracle's Woodbury and dense forms."""
    r = workloads.rng(43)
    for (n, k, lr) in [(64, 16, 1e-2), (200, 30, 0.3), (128, 64, 1.0), (96, 96, 2.0)]:
        W = _orth(r, n, k)
        V = orc.project_tangent(W, r.standard_normal((n, k)))
        c = lr / 2
        P, Q, R = W.T @ V, W.T @ W, V.T @ V
        C = np.block([[np.eye(k) + c * P, c * Q], [-c * R, np.eye(k) - c * P.T]])
        z = np.linalg.solve(C, np.concatenate([c * Q, -c * P.T], axis=0))
        W_new = W - 2 * (V @ z[:k] + W @ z[k:])
        assert np.max(np.abs(W_new - orc.cayley_woodbury(W, V, lr))) < 1e-12
        assert np.max(np.abs(W_new - orc.cayley_dense(W, V, lr))) < 1e-12
        assert orc.orthogonality_error(W_new) < 1e-12


def test_cayley_first_order_and_small_lr_limit():
    r = workloads.rng(43)
    n, k = 40, 8
    W = _orth(r, n, k)
    V = orc.project_tangent(W, r.standard_normal((n, k)))
    assert np.max(np.abs(orc.cayley_woodbury(W, V, 1e-12) - W)) < 1e-10
    AW = V @ (W.T @ W) - W @ (V.T @ W)
    h = 1e-6
    fd = (orc.cayley_woodbury(W, V, h) - W) / h
    assert np.allclose(fd, -AW, atol=1e-5)


def test_stiefel_toy_run_stays_on_manifold():
    toy = GOLDEN["stiefel_toy"]
    r = workloads.rng(44)
    W = _orth(r, toy["n"], toy["k"])
    for _ in range(toy["steps"]):
        W = orc.stiefel_cayley_step(W, r.standard_normal(W.shape), toy["lr"])
    assert orc.orthogonality_error(W) < 1e-12


# --------------------------------------------------------------------- MuonCayley

def test_ema_momentum_special_cases():
    r = workloads.rng(51)
    M0, G = r.standard_normal((6, 4)), r.standard_normal((6, 4))
    assert np.array_equal(orc.ema_momentum(M0, G, 0.0), G)
    assert np.array_equal(orc.ema_momentum(M0, G, 1.0), M0)
    # a constant gradient is a fixed point of the average
    assert np.allclose(orc.ema_momentum(G, G, 0.9), G)


def test_center_columns_is_the_column_mean_projection():
    r = workloads.rng(52)
    M = r.standard_normal((7, 5)) + np.arange(5)          # distinct column offsets
    C = orc.center_columns(M)
    assert np.allclose(C.sum(axis=0), 0.0, atol=1e-12)     # every column sums to zero
    assert np.allclose(orc.center_columns(C), C)           # idempotent
    assert np.allclose(M - C, np.ones((7, 1)) @ M.mean(axis=0, keepdims=True))   # removes a rank-1 row-constant part
    assert np.allclose(orc.center_columns(np.ones((7, 1)) @ r.standard_normal((1, 5))), 0.0)


def test_muon_cayley_step_stays_on_manifold_and_reduces_to_stiefel_step():
    r = workloads.rng(53)
    n, k = 48, 12
    W = _orth(r, n, k)
    M = np.zeros((n, k))
    for _ in range(20):
        G = r.standard_normal((n, k))
        W, M = orc.muon_cayley_step(W, G, M, lr=3e-3, beta=0.9)
    assert orc.orthogonality_error(W) < 1e-12
    # beta = 0, no centering: exactly the plain projected Cayley step of the gradient
    G = r.standard_normal((n, k))
    W1, M1 = orc.muon_cayley_step(W, G, np.zeros((n, k)), lr=0.05, beta=0.0, center=False)
    assert np.allclose(W1, orc.stiefel_cayley_step(W, G, 0.05), atol=1e-14) and np.array_equal(M1, G)


def test_muon_cayley_step_on_a_wide_parameter_keeps_rows_orthonormal():
    """§4.4 / §6.1: a parameter with fewer rows than columns is updated as its transpose.
    Its rows stay orthonormal, and the centring then removes each row's mean: a gradient
    that is constant along every row has no direction left and leaves W unchanged."""
    r = workloads.rng(54)
    rows, cols = 12, 48
    W = _orth(r, cols, rows).T
    W0 = W.copy()
    M = np.zeros((rows, cols))
    for _ in range(20):
        G = r.standard_normal((rows, cols))
        W, M = orc.muon_cayley_step(W, G, M, lr=3e-3, beta=0.9)
    assert np.max(np.abs(W @ W.T - np.eye(rows))) < 1e-12
    assert np.max(np.abs(W - W0)) > 1e-3
    G_rows = r.standard_normal((rows, 1)) @ np.ones((1, cols))
    W1, M1 = orc.muon_cayley_step(W, G_rows, np.zeros((rows, cols)), lr=0.5, beta=0.0, center=True)
    assert np.array_equal(M1, G_rows) and np.allclose(W1, W, atol=1e-15)
    # the same gradient without centring does move W
    W2, _ = orc.muon_cayley_step(W, G_rows, np.zeros((rows, cols)), lr=0.5, beta=0.0, center=False)
    assert np.max(np.abs(W2 - W)) > 1e-3


@pytest.mark.parametrize("rows,cols", [(24, 40), (40, 24)])
def test_full_step_on_a_rank_one_gradient_has_a_closed_form(rows, cols):
    """beta = 0 and M0 = 0 make M1 = G.  With G = u v^T on entries +-2^e, the bf16 cast is exact and
    G has one singular value, so the Frobenius pre-scale makes it 1 and Newton-Schulz returns
    phi_5(1) u^ v^T (u^, v^ unit vectors), whatever the orientation.  The step is then
    W1 = (1 - lr wd) W0 - lr * 0.2 sqrt(max(rows, cols)) * phi_5(1) u^ v^T.  This pins the whole
    chain (momentum, cast, pre-scale, iteration, transpose handling, scale, decay order) at
    once; phi_5(1) = 0.69644 is the rank-1 worked value."""
    r = workloads.rng(57)
    u = np.where(r.random(rows) < 0.5, -1.0, 1.0) * 2.0 ** r.integers(-3, 3, rows)
    v = np.where(r.random(cols) < 0.5, -1.0, 1.0) * 2.0 ** r.integers(-3, 3, cols)
    G = np.outer(u, v) * 2.0 ** -10
    assert np.array_equal(orc.round_to_bf16(G), G)
    W0 = orc.round_to_bf16(r.standard_normal((rows, cols)) * 0.02)
    lr, wd = 0.02, 0.1
    out = orc.muon_step(W0, G, np.zeros((rows, cols)), lr=lr, beta=0.0, weight_decay=wd)
    phi = 0.69644
    uh, vh = u / np.linalg.norm(u), v / np.linalg.norm(v)
    assert np.allclose(out["O"], phi * np.outer(uh, vh), atol=1e-5)
    want = (1 - lr * wd) * W0 - lr * 0.2 * np.sqrt(max(rows, cols)) * phi * np.outer(uh, vh)
    assert np.max(np.abs(out["W1_exact"] - want)) < 1e-6
