"""The threaded oracle driver (oracle/pool.py) against the plain
single-threaded oracle: the forward is the same ray by ray, the back
projection the same up to the order in which view ranges are summed."""
import numpy as np

import oracle
from oracle import pool as oracle_pool
from tests.helpers import small_geometries


def test_pool_matches_single_threaded_oracle():
    for name, g in small_geometries().items():
        rng = np.random.default_rng(5)
        vol = rng.random(g.vol_shape).astype(np.float32)
        sino = rng.random(g.sino_shape).astype(np.float32)
        np.testing.assert_array_equal(oracle_pool.forward(g, vol, threads=3), oracle.forward(g, vol))
        ref = oracle.back(g, sino)
        got = oracle_pool.back(g, sino, threads=3)
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max(), err_msg=name)
        got2 = oracle_pool.back(g, sino, power=2, threads=2)
        np.testing.assert_allclose(got2, oracle.back(g, sino, power=2), rtol=1e-12,
                                   atol=1e-12 * np.abs(got2).max(), err_msg=name)
