"""The diagonal fold of a quantized product chosen by a geometric program, float64.
Test infrastructure only (imported by tests/ and the bench's CPU legs, never by the
library).

"Contraction-Gauge Preconditioning for Quantized Matrix Multiplication" (abstract):
for C = A B with both factors quantized and independent zero-mean entrywise errors
of known variance fields V_A, V_B, the expected squared product error is

    E ||(A + E_A)(B + E_B) - A B||_F^2
        = sum_{i,j,k} ( V_A[i,k] B[k,j]^2 + A[i,k]^2 V_B[k,j] + V_A[i,k] V_B[k,j] ),

exact for non-overloading subtractive dither. The product is unchanged by a gauge
A B = (A T)(T^-1 B); within positive diagonal gauges T = diag(t) (folds), a
geometric program gives the globally optimal shared fold.

Reading for the SVDQuant linear ("SVDQuant Smoothing, Low-rank and Residual
Quantization", Formula item 1): A = x [m, K], B = W [K, n], and the fold is the
smoothing, t = 1 / scale (X_hat = x / scale, the smoothed weight scale * W). The
quantizer is the per-tensor grid of Formula item 3, step Delta = max|operand| / qmax;
under the dither model every element of an operand has error variance Delta^2 / 12.
With the channel statistics a_k = max_i |x_ik|, alpha_k = sum_i x_ik^2,
b_k = max_j |W_kj|, beta_k = sum_j W_kj^2 the expected error of fold t is

    E(t) = m U^2 / (12 q^2) sum_k beta_k / t_k^2 + n V^2 / (12 q^2) sum_k alpha_k t_k^2
           + K m n U^2 V^2 / (144 q^4),   U = max_k a_k t_k,  V = max_k b_k / t_k,

a posynomial in (t, U, V) under the monomial constraints a_k t_k / U <= 1 and
b_k / (t_k V) <= 1: a geometric program. It is invariant under t -> c t, so the oracle
fixes U = 1. Channels with a_k = 0 or b_k = 0 carry no product term and are left out
of the program (reading); they take the geometric mean of the other t_k, moved only
as far as needed to keep U = 1 and V as the program chose it.

The oracle solves the program in its convex log form with a general-purpose solver
(scipy SLSQP over y = log t and v = log V), so it shares no method with the library's
solver.
"""

from __future__ import annotations

import numpy as np

from .svdquant import qmax_of


def channel_stats(x, W):
    """(a, alpha, b, beta): per input channel k, max|x[:, k]|, sum x[:, k]^2,
    max|W[k, :]|, sum W[k, :]^2 (float64)."""
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    return (np.max(np.abs(x), axis=0), np.sum(x * x, axis=0),
            np.max(np.abs(W), axis=1), np.sum(W * W, axis=1))


def dither_error(A, B, var_a, var_b) -> float:
    """The identity's right-hand side for variance fields var_a [m, K], var_b [K, n]."""
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    va = np.broadcast_to(np.asarray(var_a, dtype=np.float64), A.shape)
    vb = np.broadcast_to(np.asarray(var_b, dtype=np.float64), B.shape)
    return float(np.sum(va @ (B * B)) + np.sum((A * A) @ vb) + np.sum(va @ vb))


def fold_error(stats, t, m: int, n: int, bits: int) -> float:
    """E(t): the dither-model expected squared error of the folded product with
    per-tensor grids of `bits` on both operands."""
    a, alpha, b, beta = (np.asarray(s, dtype=np.float64) for s in stats)
    t = np.asarray(t, dtype=np.float64)
    q = float(qmax_of(bits))
    K = a.shape[0]
    U = float(np.max(a * t))
    V = float(np.max(b / t))
    return (m * U * U / (12 * q * q) * float(np.sum(beta / (t * t))) +
            n * V * V / (12 * q * q) * float(np.sum(alpha * t * t)) +
            K * m * n * U * U * V * V / (144 * q ** 4))


def gp_fold(stats, m: int, n: int, bits: int, x0=None):
    """The fold t minimising fold_error, normalised to max_k a_k t_k = 1, by SLSQP on
    the convex log form of the geometric program."""
    from scipy.optimize import minimize

    a, alpha, b, beta = (np.asarray(s, dtype=np.float64) for s in stats)
    q = float(qmax_of(bits))
    live = (a > 0) & (b > 0)
    K = a.shape[0]
    la, lb = np.log(a[live]), np.log(b[live])
    al, be = alpha[live], beta[live]
    c1, c2, c3 = m / (12 * q * q), n / (12 * q * q), K * m * n / (144 * q ** 4)

    # variables z = (y_1 .. y_L, v): t = exp(y), V = exp(v), U = 1
    def f(z):
        y, v = z[:-1], z[-1]
        terms = np.array([c1 * np.sum(be * np.exp(-2 * y)), c2 * np.exp(2 * v) * np.sum(al * np.exp(2 * y)),
                          c3 * np.exp(2 * v)])
        return float(np.log(np.sum(terms)))

    def grad(z):
        y, v = z[:-1], z[-1]
        t1 = c1 * be * np.exp(-2 * y)
        t2 = c2 * np.exp(2 * v) * al * np.exp(2 * y)
        t3 = c3 * np.exp(2 * v)
        tot = np.sum(t1) + np.sum(t2) + t3
        g = np.empty_like(z)
        g[:-1] = (-2 * t1 + 2 * t2) / tot
        g[-1] = (2 * np.sum(t2) + 2 * t3) / tot
        return g

    L = int(live.sum())
    # U = 1: y_k + log a_k <= 0;  V >= b_k / t_k: log b_k - y_k - v <= 0
    A1 = np.hstack([-np.eye(L), np.zeros((L, 1))])
    A2 = np.hstack([np.eye(L), np.ones((L, 1))])
    cons = [{"type": "ineq", "fun": lambda z: A1 @ z - la, "jac": lambda z: A1},
            {"type": "ineq", "fun": lambda z: A2 @ z - lb, "jac": lambda z: A2}]
    if x0 is None:
        y0 = -la - np.log(2.0)
        v0 = np.max(lb - y0) + np.log(2.0)
        x0 = np.concatenate([y0, [v0]])
    res = minimize(f, x0, jac=grad, constraints=cons, method="SLSQP",
                   options={"maxiter": 2000, "ftol": 1e-15})
    y = res.x[:-1]
    t = np.ones(K)
    t[live] = np.exp(y)
    # channels without a product term take the geometric mean of the others, moved
    # only as far as needed to keep U = 1 (a_k > 0) and V unchanged (b_k > 0)
    gm = float(np.exp(np.mean(y))) if L else 1.0
    V = float(np.max(b[live] / t[live])) if L else 1.0
    for k in np.nonzero(~live)[0]:
        tk = gm
        if a[k] > 0:
            tk = min(tk, 1.0 / a[k])
        if b[k] > 0:
            tk = max(tk, b[k] / V)
        t[k] = tk
    return t


def alpha_fold(stats, alpha: float):
    """The fold of the migration scale of strength alpha (t = 1 / scale)."""
    a, _, b, _ = (np.asarray(s, dtype=np.float64) for s in stats)
    sa = np.where(a > 0, np.power(np.where(a > 0, a, 1.0), alpha), 1.0)
    sb = np.where(b > 0, np.power(np.where(b > 0, b, 1.0), 1.0 - alpha), 1.0)
    return sb / sa
