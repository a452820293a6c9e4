"""The library's host-only timestep schedule (fvattn_timestep_params, no
device call) against the oracle's, over a grid of steps and settings."""
import itertools
import os

import pytest

from oracle import fvattn_oracle as O

LIB = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_spatiotemporal_b200", "libfvattn.so")


@pytest.mark.skipif(not os.path.exists(LIB), reason="libfvattn.so not built")
def test_timestep_params_match_the_oracle():
    from block_sparse_spatiotemporal_b200 import fvattn as F
    for num_steps, dense, (p0, p1), (k0, k1) in itertools.product(
            (1, 2, 10, 50), (0, 3), ((0.99, 0.9), (0.95, 0.5), (1.0, 1.0)), ((8, 8), (2, 16), (16, 4))):
        for step in range(num_steps):
            p, k = F.timestep_params(step, num_steps, p0, p1, k0, k1, dense)
            rp, rk = O.timestep_params(step, num_steps, p0, p1, k0, k1, dense)
            assert abs(p - rp) <= 1e-6 and k == rk, (num_steps, dense, p0, p1, k0, k1, step)


@pytest.mark.skipif(not os.path.exists(LIB), reason="libfvattn.so not built")
def test_timestep_params_reject_bad_steps():
    from block_sparse_spatiotemporal_b200 import fvattn as F
    for bad in ((-1, 10), (10, 10), (0, 0)):
        with pytest.raises(F.FvattnError):
            F.timestep_params(bad[0], bad[1], 0.9, 0.5, 8, 8)
