"""The FMA-pipe 2^x of kernel option bit 3 (exp2_fma2) on the GPU against
float64 2^x and against the special-function unit's ex2.approx: relative
error within the fitted polynomial's bound (1.8e-7, plus the float32 FMA
rounding of the reduction) over the whole normal range, exact powers of
two at integers and 1 at 0, finite and tiny below the clamp, finite and
huge above it."""
import numpy as np
import pytest
import torch

from selective_state_space_31_b200 import binding as bnd

pytestmark = pytest.mark.gpu


def test_exp2_fma_against_float64_and_ex2_approx():
    rng = np.random.default_rng(21)
    x = np.concatenate([np.linspace(-124.9, 126.9, 1_000_001),
                        rng.uniform(-40.0, 0.0, 1_000_000),       # the scan's usual arguments
                        np.arange(-125, 128), [0.0, -0.5, 0.5, -1e-30, 1e-30]]).astype(np.float32)
    y_fma, y_sfu = bnd.probe_exp2(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    yf = y_fma.cpu().numpy().astype(np.float64)
    ys = y_sfu.cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.all(np.isfinite(yf))
    rel = np.abs(yf - ref) / ref
    assert rel.max() < 2.5e-7, rel.max()
    # against the special-function unit (its own error is about 2^-22)
    assert (np.abs(yf - ys) / ys).max() < 6e-7
    ints = np.arange(-125, 128)
    k = len(x) - 5 - len(ints)
    assert np.array_equal(yf[k:k + len(ints)], np.exp2(ints.astype(np.float64)))
    assert yf[-5] == 1.0 and yf[-2] == 1.0 and yf[-1] == 1.0


def test_exp2_fma_outside_the_normal_range():
    x = np.array([-126.0, -150.0, -1e4, -np.inf, 127.5, 200.0, 1e4], dtype=np.float32)
    y_fma, y_sfu = bnd.probe_exp2(torch.from_numpy(x).cuda())
    yf = y_fma.cpu().numpy()
    assert np.all(np.isfinite(yf))
    assert np.all((yf[:4] >= 0) & (yf[:4] <= 2.0 ** -124))
    assert np.all(yf[4:] >= 2.0 ** 126)

