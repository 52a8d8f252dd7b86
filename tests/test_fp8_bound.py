"""CPU check of the FP8 forward's derived tolerance (the bound the GPU parity test applies):
an fp64 model of the one 8-bit rounding inside the kernel — each softmax weight
p_j = 2^(x_j - m + 6), with m any reference maximum in [max x - 2.5, max x] (the lazy
refresh window), rounded to E4M3 by PyTorch's float8_e4m3fn cast, and O = sum_j p~_j v_j /
sum_j p~_j — must stay within

    2^-4/(1 - 2^-4) * sum_j w_j |v_j - O_ref| + 2^-16/(1 - 2^-4) * sum_j |v_j - O_ref| / sum_j 2^(x_j - max x)

of the exact O_ref for every row, over flat, peaky and wide score distributions.  The
model uses no code of the CUDA library."""

import numpy as np
import pytest
import torch

EPS8 = 2.0 ** -4


def _row_case(rng, n, spread, lazy):
    x = rng.standard_normal(n) * spread                 # log2-domain scores
    v = rng.standard_normal((n, 16)) * 2.0
    mx = x.max()
    m = mx - lazy                                       # reference maximum, lazily refreshed
    p = np.exp2(x - m + 6.0)
    p8 = torch.from_numpy(p).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    o_model = (p8 @ v) / p8.sum()
    w = np.exp2(x - mx)
    o_ref = (w @ v) / w.sum()
    dev = np.abs(v - o_ref[None, :])
    b1 = EPS8 / (1 - EPS8) * ((w / w.sum()) @ dev)
    b2 = 2.0 ** -16 / (1 - EPS8) * dev.sum(axis=0) / w.sum()
    return np.abs(o_model - o_ref), b1 + b2


@pytest.mark.parametrize("spread", [0.5, 3.0, 12.0, 40.0])
@pytest.mark.parametrize("lazy", [0.0, 1.3, 2.5])
def test_model_error_within_the_derived_bound(spread, lazy):
    rng = np.random.default_rng(int(spread * 10) + int(lazy * 100))
    worst = 0.0
    for n in (1, 2, 17, 128, 1000, 4096):
        for _ in range(8):
            err, bound = _row_case(rng, n, spread, lazy)
            assert np.all(err <= bound * (1 + 1e-12) + 1e-15), (n, spread, lazy, (err / bound).max())
            worst = max(worst, float((err / np.maximum(bound, 1e-300)).max()))
    assert worst > 0.0


def test_bound_is_not_vacuous():
    # the modelled rounding uses a sizeable part of the bound: it is not loose by orders of
    # magnitude, so the parity test that applies it can still fail
    rng = np.random.default_rng(5)
    ratios = []
    for _ in range(50):
        err, bound = _row_case(rng, 512, 3.0, 1.0)
        ratios.append(float((err / bound).max()))
    assert max(ratios) > 0.2
