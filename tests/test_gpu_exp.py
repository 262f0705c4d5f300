"""The stochastic verify's fp64 exponential (Tang's table-driven method,
arguments <= 0) against CUDA's exp and numpy's on the host."""
import numpy as np
import pytest
import torch

import step_flow_map_b200 as fmb

pytestmark = pytest.mark.gpu


def _run(e_np):
    e = torch.from_numpy(e_np).cuda()
    mine, ref = torch.empty_like(e), torch.empty_like(e)
    fmb.fm_selftest_exp(e, mine, ref)
    torch.cuda.synchronize()
    return mine.cpu().numpy(), ref.cpu().numpy()


def test_exp_matches_cuda_and_numpy_within_two_ulp():
    rng = np.random.default_rng(5)
    e = np.concatenate([
        -rng.uniform(0.0, 700.0, 1_000_000),
        -rng.uniform(0.0, 1.0, 200_000),
        -rng.exponential(1e-6, 20_000),
        -np.arange(0, 700, dtype=np.float64) * np.log(2.0) / 32.0,   # table knots
        np.array([0.0, -0.0, -1e-300, -699.999]),
    ])
    mine, ref = _run(e)
    host = np.exp(e)
    ulp = np.spacing(host)
    assert np.all(np.abs(mine - ref) <= 2 * np.spacing(ref))
    assert np.all(np.abs(mine - host) <= 2 * ulp)
    assert mine[-4] == 1.0 and mine[-3] == 1.0


def test_exp_special_values():
    e = np.array([-700.5, -1e4, -np.inf, np.nan], dtype=np.float64)
    mine, _ = _run(e)
    assert mine[0] == 0.0 and mine[1] == 0.0 and mine[2] == 0.0
    assert np.isnan(mine[3])
