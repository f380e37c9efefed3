"""Plain fp64 CPU oracle for the Muon optimizer step and its Stiefel/Cayley variant.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: it is used by ``tests/``, by ``__graft_entry__.smoke()``
(to check one small GPU result) and by the ``cpu_baseline`` / reference arm of
``bench.py``.  It shares no code, constants table or helper with the CUDA
library; the two meet only in the seeded input generators, which hold none of
the method's arithmetic.

Every function is written out in the order and notation of the source pages,
in float64 with NumPy, without blocking, fusion or reordering.  Sources:

* "Muon优化器" (Muon optimizer), linsight.cn/f25d614e.html -- sections
  "Muon 的核心思想" (msign), "Newton-Schulz 迭代" (NS iteration, coefficients,
  ``zeropower_via_newtonschulz``), "缩放因子" (the four update scalings) and
  "Muon 算法伪代码与 PyTorch 实现" (the ``Muon.step`` loop: momentum, Nesterov,
  NS, scale, decoupled weight decay).
* "Muon 在 Stiefel 流形上的精确闭式更新" (Muon on the Stiefel manifold admits
  an exact closed-form update), mlqm.cn/news/1339166 -- §1.3 tangent
  projection, §3.1-3.2 Cayley retraction, §6.2 the Woodbury rank-2k form.
* prism.simon-ai.net/article/8795, section "Muon的训练效率与DeepSeek V4的混合
  优化策略" -- the hybrid schedule (8 fast iterations, then 2 stabilising ones).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, invariants, library routines or brute force; none is
"parity unpinned".
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# Coefficients and schedules
# ---------------------------------------------------------------------------

#: (a, b, c) tuned for square matrices and T = 5 steps.  Muon optimizer page,
#: "Newton-Schulz 迭代": the empirically optimised coefficients.
KJ_COEFFS = (3.4445, -4.7750, 2.0315)

#: (a, b, c) from the second-order Taylor expansion of t^(-1/2) at t = 1,
#: t^(-1/2) ~ (15 - 10 t + 3 t^2) / 8.  Muon optimizer page, "NS 迭代的数学原理
#: 与系数来源".  The only printed set with phi(1) = 1 and phi'(1) = 0, used as
#: the stabilising stage of the hybrid schedule (a reading: the hybrid
#: schedule's own coefficients are not printed on any page).
TEXTBOOK_COEFFS = (1.875, -1.25, 0.375)

#: Frobenius pre-scaling epsilon, added to the norm (not to its square).
#: Muon optimizer page, ``zeropower_via_newtonschulz(G, steps=5, eps=1e-7)``.
NS_EPS = 1e-7


def fixed_schedule(steps: int = 5, coeffs=KJ_COEFFS):
    """T identical iterations (the page's ``steps`` loop)."""
    return [tuple(coeffs)] * int(steps)


def hybrid_schedule(n_fast: int = 8, n_stable: int = 2,
                    fast=KJ_COEFFS, stable=TEXTBOOK_COEFFS):
    """Hybrid NS: ``n_fast`` iterations that push singular values toward 1
    quickly, then ``n_stable`` that hold them at 1 (prism.simon-ai.net, DeepSeek
    V4 section: 8 fast then 2 stabilising)."""
    return [tuple(fast)] * int(n_fast) + [tuple(stable)] * int(n_stable)


# ---------------------------------------------------------------------------
# Storage rounding (the method keeps M in fp32 and casts it to bf16)
# ---------------------------------------------------------------------------

def round_to_f32(x):
    """Round to the nearest float32 and return as float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_to_bf16(x):
    """Round-to-nearest-even from float32 to bfloat16, returned as float64.

    The value is first taken to float32 (the storage type of the momentum
    buffer and of the update arithmetic), then its low 16 bits are dropped with
    ties to even -- the definition of the ``.bfloat16()`` cast the Muon page's
    ``zeropower_via_newtonschulz`` applies.  NaN stays NaN, +-inf stays inf.
    """
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    bits = x32.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    out = (rounded & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    nan = np.isnan(x32)
    if np.any(nan):
        out = np.where(nan, np.float32(np.nan), out)
    return out.astype(np.float64)


# ---------------------------------------------------------------------------
# Muon step (Muon optimizer page, "Muon 算法伪代码与 PyTorch 实现")
# ---------------------------------------------------------------------------

def momentum(M0, G, beta: float, nesterov: bool = False):
    """Heavy-ball momentum ``buf.mul_(beta).add_(g)``: M1 = beta*M0 + G.

    With Nesterov the matrix handed to Newton-Schulz is beta*M1 + G, else M1.
    Returns (M1, g_update).
    """
    M0 = np.asarray(M0, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    M1 = beta * M0 + G
    g_update = beta * M1 + G if nesterov else M1
    return M1, g_update


def ns_input(g_update, fp32_mode: bool = False):
    """The matrix Newton-Schulz starts from.

    bf16 mode (the page): ``X = G.bfloat16()`` of the fp32 momentum buffer.
    fp32 mode: the fp32 buffer itself (no cast)."""
    if fp32_mode:
        return round_to_f32(g_update)
    return round_to_bf16(g_update)


def frobenius_prescale(X, eps: float = NS_EPS):
    """X / (||X||_F + eps), so that sigma_max(X) <= 1 (||.||_2 <= ||.||_F)."""
    X = np.asarray(X, dtype=np.float64)
    return X / (np.sqrt(np.sum(X * X)) + eps)


def newton_schulz(X0, schedule, eps: float = NS_EPS):
    """``zeropower_via_newtonschulz`` in fp64, with per-iteration (a, b, c).

    Steps, in the page's order: Frobenius pre-scale; transpose when rows >
    cols so that X X^T is the small Gram matrix; per iteration
    A = X X^T, B = b A + c A A, X = a X + B X; transpose back.
    No rounding anywhere (the bf16 casts of the page are the GPU's business).
    """
    X = frobenius_prescale(X0, eps)
    transpose = X.shape[0] > X.shape[1]
    if transpose:
        X = X.T
    for (a, b, c) in schedule:
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    if transpose:
        X = X.T
    return np.ascontiguousarray(X)


def msign_svd(M):
    """Exact matrix sign msign(M) = U V^T from the thin SVD M = U S V^T
    (Muon optimizer page, "Muon 的核心思想")."""
    U, _, Vt = np.linalg.svd(np.asarray(M, dtype=np.float64), full_matrices=False)
    return U @ Vt


SCALE_MODES = ("moonlight", "kellerjordan", "mup", "naive")


def scale_factor(rows: int, cols: int, mode: str = "moonlight") -> float:
    """Update scale for W in R^{d_out x d_in} (PyTorch Linear layout, rows =
    d_out, cols = d_in).  Muon optimizer page, "缩放因子" table and
    ``Muon.get_scale``."""
    d_out, d_in = float(rows), float(cols)
    if mode == "moonlight":
        return 0.2 * np.sqrt(max(d_out, d_in))
    if mode == "kellerjordan":
        return float(np.sqrt(max(1.0, d_out / d_in)))
    if mode == "mup":
        return float(np.sqrt(d_out / d_in))
    if mode == "naive":
        return 1.0
    raise ValueError(f"unknown scale mode {mode!r}")


def muon_update(W0, O, lr: float, weight_decay: float, scale: float):
    """Decoupled weight decay then the step, in the page's order:
    ``p.mul_(1 - lr*wd)`` then ``p.add_(scale*O, alpha=-lr)``."""
    W0 = np.asarray(W0, dtype=np.float64)
    return (1.0 - lr * weight_decay) * W0 - lr * (scale * np.asarray(O, dtype=np.float64))


def muon_step(W0, G, M0, *, lr: float, beta: float = 0.95, weight_decay: float = 0.0,
              nesterov: bool = False, scale_mode: str = "moonlight", schedule=None,
              fp32_mode: bool = False, eps: float = NS_EPS, w_dtype: str = "bf16"):
    """One full Muon step on one matrix.

    Returns a dict with M1 (fp64; the GPU stores it as fp32), X0 (the NS
    input), O (the fp64 NS output), scale, W1_exact (fp64) and W1 (rounded to
    the weight dtype: bf16 RNE of the fp32 result, or fp32)."""
    if schedule is None:
        schedule = fixed_schedule(5)
    M1, g_upd = momentum(M0, G, beta, nesterov)
    X0 = ns_input(g_upd, fp32_mode)
    O = newton_schulz(X0, schedule, eps) if len(schedule) else frobenius_prescale(X0, eps)
    rows, cols = np.shape(W0)
    s = scale_factor(rows, cols, scale_mode)
    W1_exact = muon_update(W0, O, lr, weight_decay, s)
    W1 = round_to_bf16(W1_exact) if w_dtype == "bf16" else round_to_f32(W1_exact)
    return {"M1": M1, "X0": X0, "O": O, "scale": s, "W1_exact": W1_exact, "W1": W1}


# ---------------------------------------------------------------------------
# Stiefel variant (mlqm.cn/news/1339166)
# ---------------------------------------------------------------------------

def project_tangent(W, G):
    """§1.3 / §3.2: G_t = G - W sym(W^T G), sym(S) = (S + S^T)/2."""
    W = np.asarray(W, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    S = W.T @ G
    return G - W @ (0.5 * (S + S.T))


def cayley_dense(W, V, lr: float):
    """§3.2: A = V W^T - W V^T (n x n skew), c = lr/2,
    W_new = (I + cA)^(-1) (I - cA) W, by a dense n x n solve."""
    W = np.asarray(W, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    n = W.shape[0]
    c = lr / 2.0
    A = V @ W.T - W @ V.T
    I = np.eye(n)
    return np.linalg.solve(I + c * A, (I - c * A) @ W)


def cayley_woodbury(W, V, lr: float):
    """§6.2: the same retraction through the rank-2k factorisation A = U B,
    U = [V, W] (n x 2k), B = [W^T; -V^T] (2k x n):
    C = I_2k + c B U; b = W - c U (B W); z = C^(-1) (B b); W_new = b - c U z."""
    W = np.asarray(W, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    k = W.shape[1]
    c = lr / 2.0
    U = np.concatenate([V, W], axis=1)
    B = np.concatenate([W.T, -V.T], axis=0)
    C = np.eye(2 * k) + c * (B @ U)
    b = W - c * (U @ (B @ W))
    z = np.linalg.solve(C, B @ b)
    return b - c * (U @ z)


def stiefel_cayley_step(W, G, lr: float, woodbury: bool = True):
    """Project G onto the tangent space at W, then retract with Cayley."""
    V = project_tangent(W, G)
    return cayley_woodbury(W, V, lr) if woodbury else cayley_dense(W, V, lr)


def orthogonality_error(W):
    """max |W^T W - I| (§5.1's check, in max-norm)."""
    W = np.asarray(W, dtype=np.float64)
    return float(np.max(np.abs(W.T @ W - np.eye(W.shape[1]))))


# ---------------------------------------------------------------------------
# MuonCayley optimizer update (mlqm.cn/news/1339166, §3.3 and §4.3)
# ---------------------------------------------------------------------------

def ema_momentum(M0, G, beta: float):
    """§3.3 / §4.3 ``buf.mul_(momentum).add_(grad, alpha=1 - momentum)``:
    M1 = beta*M0 + (1 - beta)*G."""
    return beta * np.asarray(M0, dtype=np.float64) + (1.0 - beta) * np.asarray(G, dtype=np.float64)


def center_columns(M):
    """§4.3 ``buf - buf.mean(dim=0, keepdim=True)``: subtract each column's mean over the
    rows.  (The §3.3 prose says row mean; the printed code, which is what runs, takes
    dim=0 -- the reading this oracle follows.)"""
    M = np.asarray(M, dtype=np.float64)
    return M - M.mean(axis=0, keepdims=True)


def muon_cayley_step(W, G, M0, lr: float, beta: float, center: bool = True):
    """One MuonCayley update in the order of §4.3: EMA momentum, centering, tangent
    projection of the centred momentum, Cayley retraction (Woodbury form).
    Returns (W1, M1).

    A wide W (fewer rows than columns) cannot be column-orthonormal; §4.4 and §6.1 say
    to transpose such a parameter, update it on the manifold and transpose it back.  The
    whole step then runs on W^T, G^T, M^T (so the centring takes each row's mean of the
    caller's M) and the results are transposed back: W stays row-orthonormal."""
    if np.shape(W)[0] < np.shape(W)[1]:
        W1t, M1t = muon_cayley_step(np.asarray(W).T, np.asarray(G).T, np.asarray(M0).T, lr, beta, center)
        return W1t.T, M1t.T
    M1 = ema_momentum(M0, G, beta)
    D = center_columns(M1) if center else M1
    V = project_tangent(W, D)
    return cayley_woodbury(W, V, lr), M1
