"""FP64 reference solvers on the oracle's dense system matrix.

TEST INFRASTRUCTURE ONLY (imported by the tests, never by the library).

Both follow diffct "Execution", section "Numerical solver API":
  * the residual history holds the initial residual ||y - A x0|| and one
    value per completed iteration;
  * convergence means ||y - A x|| <= atol + rtol ||y||, checked on the
    initial iterate too;
  * SIRT takes a relaxation factor and an optional nonnegativity clamp, and
    reuses the residual of the previous history entry for its next update.

CGLS is the conjugate-gradient method on the normal equations A^T A x =
A^T y in its least-squares form (Hestenes-Stiefel recurrences on r = y - Ax
and s = A^T r).  SIRT is x <- x + lambda C A^T R (y - A x) with R and C the
reciprocal row and column sums of A (zero where a sum is zero).
"""
from __future__ import annotations

import numpy as np


def _converged(res, ynorm, atol, rtol):
    return res <= atol + rtol * ynorm


def dense_ops(A):
    """(forward, adjoint) callables of a dense matrix."""
    A = np.asarray(A, dtype=np.float64)
    return (lambda x: A @ x), (lambda y: A.T @ y), A.shape[1]


def _ops(A):
    return A if isinstance(A, tuple) else dense_ops(A)


def cgls(A, y, iterations, x0=None, atol=0.0, rtol=0.0):
    """A: a dense matrix or a (forward, adjoint, n_unknowns) triple of
    callables on flat FP64 vectors.  Returns (x, history, converged)."""
    fwd, adj, n = _ops(A)
    y = np.asarray(y, dtype=np.float64).reshape(-1)
    x = np.zeros(n) if x0 is None else np.asarray(x0, dtype=np.float64).reshape(-1).copy()
    ynorm = float(np.linalg.norm(y))
    r = y - fwd(x)
    history = [float(np.linalg.norm(r))]
    if _converged(history[0], ynorm, atol, rtol):
        return x, history, True
    s = adj(r)
    p = s.copy()
    gamma = float(s @ s)
    for _ in range(iterations):
        if gamma == 0.0:
            break
        q = fwd(p)
        delta = float(q @ q)
        if delta == 0.0:
            break
        alpha = gamma / delta
        x += alpha * p
        r -= alpha * q
        s = adj(r)
        gamma_new = float(s @ s)
        history.append(float(np.linalg.norm(r)))
        if _converged(history[-1], ynorm, atol, rtol):
            return x, history, True
        p = s + (gamma_new / gamma) * p
        gamma = gamma_new
    return x, history, False


def sirt_weights(A):
    """Reciprocal row sums R (per ray) and column sums C (per voxel), zero
    where a sum is zero (row sums A 1, column sums A^T 1)."""
    fwd, adj, n = _ops(A)
    rows = fwd(np.ones(n))
    cols = adj(np.ones(rows.shape[0]))
    R = np.where(rows > 0, 1.0 / np.where(rows > 0, rows, 1.0), 0.0)
    C = np.where(cols > 0, 1.0 / np.where(cols > 0, cols, 1.0), 0.0)
    return R, C


def sirt(A, y, iterations, x0=None, relaxation=1.0, nonnegative=True, atol=0.0, rtol=0.0):
    """A as for cgls.  Returns (x, history, converged)."""
    fwd, adj, n = _ops(A)
    y = np.asarray(y, dtype=np.float64).reshape(-1)
    x = np.zeros(n) if x0 is None else np.asarray(x0, dtype=np.float64).reshape(-1).copy()
    R, C = sirt_weights(A)
    ynorm = float(np.linalg.norm(y))
    r = y - fwd(x)
    history = [float(np.linalg.norm(r))]
    if _converged(history[0], ynorm, atol, rtol):
        return x, history, True
    for _ in range(iterations):
        x = x + relaxation * C * adj(R * r)
        if nonnegative:
            x = np.maximum(x, 0.0)
        r = y - fwd(x)
        history.append(float(np.linalg.norm(r)))
        if _converged(history[-1], ynorm, atol, rtol):
            return x, history, True
    return x, history, False
