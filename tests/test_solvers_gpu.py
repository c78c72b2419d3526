"""GPU solvers (ctp_solve: CGLS, SIRT) against the FP64 reference solvers
run on the oracle's operators.  Both are iterations on the same problem, so
iterates and residual histories agree to FP32 rounding amplified by the
iteration count; the problems are well conditioned to keep that small."""
import numpy as np
import pytest

import oracle
from oracle import solvers
from ray_forward_back_b200 import workloads as W
from tests.gpu_helpers import projector

pytestmark = pytest.mark.gpu


def _small():
    g = W.make_parallel(8, 8, 8, 10, 12, 12, pitch_u=0.7, pitch_v=0.7, start=0.05)
    src = g.src.copy()
    src[:, 2] = 0.35
    g.src = src
    return g


def _gpu_solve(g, y, method, iters, **kw):
    import torch
    P = projector(g)
    vol, hist, conv = P.solve(torch.from_numpy(np.ascontiguousarray(y, np.float32).reshape(g.sino_shape)).cuda(),
                              method, iters, **kw)
    torch.cuda.synchronize()
    return vol.cpu().numpy().reshape(-1).astype(np.float64), np.array(hist), conv


def test_cgls_matches_reference_iterates():
    g = _small()
    A = oracle.dense_matrix(g)
    y = np.random.default_rng(1).random(A.shape[0]).astype(np.float32)
    x_ref, h_ref, _ = solvers.cgls(A, y.astype(np.float64), 8)
    x, h, conv = _gpu_solve(g, y, "cgls", 8)
    assert len(h) == len(h_ref) == 9 and not conv
    np.testing.assert_allclose(h, h_ref, rtol=1e-5)
    assert np.linalg.norm(x - x_ref) <= 1e-4 * np.linalg.norm(x_ref)


def test_sirt_matches_reference_iterates():
    g = _small()
    A = oracle.dense_matrix(g)
    y = np.random.default_rng(2).random(A.shape[0]).astype(np.float32)
    for relax, nonneg in ((1.0, True), (0.7, False)):
        x_ref, h_ref, _ = solvers.sirt(A, y.astype(np.float64), 15, relaxation=relax, nonnegative=nonneg)
        x, h, _ = _gpu_solve(g, y, "sirt", 15, relaxation=relax, nonnegative=nonneg)
        assert len(h) == len(h_ref) == 16
        np.testing.assert_allclose(h, h_ref, rtol=1e-5)
        assert np.linalg.norm(x - x_ref) <= 1e-5 * np.linalg.norm(x_ref)
        if nonneg:
            assert x.min() >= 0.0


def test_tolerance_stops_and_initial_iterate_counts():
    import torch
    g = _small()
    A = oracle.dense_matrix(g)
    x_true = np.random.default_rng(3).random(A.shape[1]).astype(np.float32)
    y = (A @ x_true.astype(np.float64)).astype(np.float32)
    x, h, conv = _gpu_solve(g, y, "cgls", 200, rtol=1e-4)
    assert conv and len(h) < 201 and h[-1] <= 1e-4 * np.linalg.norm(y)
    assert np.linalg.norm(x - x_true) <= 1e-3 * np.linalg.norm(x_true)
    # an initial iterate that already meets the tolerance runs no iteration
    P = projector(g)
    x0 = torch.from_numpy(x_true.reshape(g.vol_shape)).cuda()
    vol, hist, conv = P.solve(torch.from_numpy(y.reshape(g.sino_shape)).cuda(), "sirt", 5, rtol=1e-3, x0=x0)
    assert conv and len(hist) == 1
    assert torch.equal(vol, x0)


def test_cgls_on_workload1_against_matrix_free_reference():
    """Workload 1 (64^3 cone, 16 views): three CGLS iterations against the
    reference CGLS on the oracle's own forward and adjoint."""
    wl = W.workload(1)
    g = wl.geom
    y = oracle.forward(g, wl.phantom()).astype(np.float32)
    fwd = lambda x: oracle.forward(g, x.reshape(g.vol_shape).astype(np.float32)).reshape(-1)
    adj = lambda s: oracle.back(g, s.reshape(g.sino_shape).astype(np.float32)).reshape(-1)
    # the reference promotes its iterates to FP32 before every projection, as the GPU stores them
    x_ref, h_ref, _ = solvers.cgls((fwd, adj, g.n_vox), y.astype(np.float64).reshape(-1), 3)
    x, h, _ = _gpu_solve(g, y, "cgls", 3)
    np.testing.assert_allclose(h, h_ref, rtol=1e-4)
    assert np.linalg.norm(x - x_ref) <= 1e-3 * np.linalg.norm(x_ref)


@pytest.mark.slow
def test_solvers_on_workload2_view_subset_against_matrix_free_reference():
    """Workload 2 at its full size (256^3 volume, 384 x 384 detector) on 12
    evenly spaced views: five CGLS and five SIRT iterations against the
    reference solvers run matrix-free on the oracle's forward and adjoint
    (spread over the host's cores).  The reference casts its iterates to FP32
    before each projection, as the GPU stores them."""
    from oracle import pool
    wl = W.workload(2)
    g = wl.geom.subset_views(np.linspace(0, wl.geom.n_views - 1, 12).round().astype(np.int64))
    y = pool.forward(g, wl.phantom()).astype(np.float32)
    fwd = lambda x: pool.forward(g, x.reshape(g.vol_shape).astype(np.float32)).reshape(-1)
    adj = lambda s: pool.back(g, s.reshape(g.sino_shape).astype(np.float32)).reshape(-1)
    y64 = y.astype(np.float64).reshape(-1)
    x_ref, h_ref, _ = solvers.cgls((fwd, adj, g.n_vox), y64, 5)
    x, h, _ = _gpu_solve(g, y, "cgls", 5)
    assert len(h) == len(h_ref) == 6
    np.testing.assert_allclose(h, h_ref, rtol=1e-4)
    assert np.linalg.norm(x - x_ref) <= 1e-3 * np.linalg.norm(x_ref)
    x_ref, h_ref, _ = solvers.sirt((fwd, adj, g.n_vox), y64, 5, relaxation=1.0, nonnegative=True)
    x, h, _ = _gpu_solve(g, y, "sirt", 5, relaxation=1.0, nonnegative=True)
    assert len(h) == len(h_ref) == 6
    np.testing.assert_allclose(h, h_ref, rtol=1e-4)
    assert np.linalg.norm(x - x_ref) <= 1e-4 * np.linalg.norm(x_ref)
    assert x.min() >= 0.0


def test_workspace_contract():
    import torch
    from ray_forward_back_b200 import ctp
    g = _small()
    P = projector(g)
    need_c = ctp.ctp_solver_workspace_bytes(P.handle, ctp.CTP_SOLVER_CGLS)
    need_s = ctp.ctp_solver_workspace_bytes(P.handle, ctp.CTP_SOLVER_SIRT)
    assert need_s > need_c > 4 * (g.n_rays + g.n_vox)
    assert ctp.ctp_solver_workspace_bytes(P.handle, 7) == 0
    y = torch.zeros(g.sino_shape, device="cuda")
    vol = torch.zeros(g.vol_shape, device="cuda")
    small = torch.empty(need_c // 2, dtype=torch.uint8, device="cuda")
    with pytest.raises(ctp.CtpError) as ei:
        ctp.ctp_solve(P.handle, y, vol, ctp.CTP_SOLVER_CGLS, 3, workspace=small)
    assert ei.value.status == ctp.CTP_ERR_INVALID_ARGUMENT
