"""Pins of the FP64 reference solvers (CPU only).

CGLS is pinned to numpy's least-squares solver (a library routine) and to
exact recovery on a consistent full-rank system; SIRT to its fixed-point
property and to nonnegativity / history / stopping rules stated by the pages.
"""
import numpy as np
import pytest

import oracle
from oracle import solvers
from ray_forward_back_b200 import workloads as W


def _system():
    """8^3 volume, 10 parallel views of a 12x12 detector: 1440 rays, 512
    unknowns, full column rank."""
    g = W.make_parallel(8, 8, 8, 10, 12, 12, pitch_u=0.7, pitch_v=0.7, start=0.05)
    src = g.src.copy()
    src[:, 2] = 0.35   # tilt out of the slices so rows couple neighbouring slices
    g.src = src
    return g, oracle.dense_matrix(g)


def test_system_has_full_column_rank():
    g, A = _system()
    assert np.linalg.matrix_rank(A) == A.shape[1]


def test_cgls_converges_to_the_least_squares_solution():
    g, A = _system()
    rng = np.random.default_rng(1)
    y = rng.random(A.shape[0])
    x, hist, _ = solvers.cgls(A, y, 200)
    x_ls = np.linalg.lstsq(A, y, rcond=None)[0]
    assert np.linalg.norm(x - x_ls) <= 1e-8 * np.linalg.norm(x_ls)
    assert hist[-1] == pytest.approx(np.linalg.norm(y - A @ x_ls), rel=1e-9)


def test_cgls_recovers_a_consistent_system_and_stops_on_tolerance():
    g, A = _system()
    rng = np.random.default_rng(2)
    x_true = rng.random(A.shape[1])
    y = A @ x_true
    x, hist, conv = solvers.cgls(A, y, 500, rtol=1e-10)
    assert conv
    assert np.linalg.norm(x - x_true) <= 1e-6 * np.linalg.norm(x_true)
    # history: initial residual plus one per iteration, the last within tolerance
    assert hist[0] == pytest.approx(np.linalg.norm(y))
    assert hist[-1] <= 1e-10 * np.linalg.norm(y)
    assert len(hist) < 501


def test_cgls_residual_is_monotone():
    g, A = _system()
    y = np.random.default_rng(3).random(A.shape[0])
    _, hist, _ = solvers.cgls(A, y, 30)
    assert all(b <= a * (1 + 1e-12) for a, b in zip(hist, hist[1:]))


def test_converged_initial_iterate_runs_no_iteration():
    g, A = _system()
    x_true = np.random.default_rng(4).random(A.shape[1])
    y = A @ x_true
    for solve in (solvers.cgls, solvers.sirt):
        x, hist, conv = solve(A, y, 10, x0=x_true, rtol=1e-9)
        assert conv and len(hist) == 1
        np.testing.assert_array_equal(x, x_true)


def test_sirt_weights_are_reciprocal_sums():
    g, A = _system()
    R, C = solvers.sirt_weights(A)
    rows, cols = A.sum(axis=1), A.sum(axis=0)
    np.testing.assert_allclose(R[rows > 0] * rows[rows > 0], 1.0)
    np.testing.assert_allclose(C * cols, 1.0)
    assert np.all(R[rows == 0] == 0)


def test_sirt_fixed_point_and_convergence():
    """A consistent system's solution is a fixed point of the SIRT map, and
    unrelaxed SIRT drives the residual of a consistent system down."""
    g, A = _system()
    x_true = np.random.default_rng(5).random(A.shape[1]) + 0.5
    y = A @ x_true
    R, C = solvers.sirt_weights(A)
    step = C * (A.T @ (R * (y - A @ x_true)))
    assert np.linalg.norm(step) <= 1e-12 * np.linalg.norm(x_true)
    x, hist, _ = solvers.sirt(A, y, 400)
    assert hist[-1] < 1e-2 * hist[0]
    assert np.linalg.norm(x - x_true) < 0.1 * np.linalg.norm(x_true)


def test_sirt_nonnegativity_and_relaxation():
    g, A = _system()
    y = np.random.default_rng(6).standard_normal(A.shape[0])   # pushes some voxels negative
    x, _, _ = solvers.sirt(A, y, 20, nonnegative=True)
    assert x.min() >= 0.0
    x2, _, _ = solvers.sirt(A, y, 20, nonnegative=False)
    assert x2.min() < 0.0
    # one step with relaxation 0.5 is half the unrelaxed step from zero
    xa, _, _ = solvers.sirt(A, y, 1, relaxation=1.0, nonnegative=False)
    xb, _, _ = solvers.sirt(A, y, 1, relaxation=0.5, nonnegative=False)
    np.testing.assert_allclose(xb, 0.5 * xa, atol=1e-14)


def test_sirt_clamp_is_the_projection_onto_nonnegative_values():
    """The nonnegativity rule is the projection max(x, 0), not any other map to
    x >= 0: from x = 0 on data y <= 0 every unclamped update is <= 0 (A, R, C
    are nonnegative), so the clamped iterate stays exactly zero, and one
    clamped step equals max(unclamped step, 0)."""
    g, A = _system()
    y = -np.random.default_rng(7).random(A.shape[0])
    x, _, _ = solvers.sirt(A, y, 5, nonnegative=True)
    assert np.count_nonzero(x) == 0
    xu, _, _ = solvers.sirt(A, y, 1, nonnegative=False)
    assert xu.max() <= 0.0 and xu.min() < 0.0
    y2 = np.random.default_rng(8).standard_normal(A.shape[0])
    one_free, _, _ = solvers.sirt(A, y2, 1, nonnegative=False)
    one_clamped, _, _ = solvers.sirt(A, y2, 1, nonnegative=True)
    np.testing.assert_array_equal(one_clamped, np.maximum(one_free, 0.0))
