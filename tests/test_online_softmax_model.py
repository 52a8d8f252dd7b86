"""CPU model of the forward kernel's online softmax as it is built (not of its code): key
tiles of 128, a reference maximum refreshed only when a tile's maximum exceeds it by more
than 8 (log2 units), p = 2^(x - m) in fp32, P rounded to bf16 for the P·V product with fp32
accumulation, O normalised by the sum of the rounded P (the ones columns) and LSE taken from
the fp32 sum of the unrounded p.  On adversarial rows — scores that climb just under the
refresh threshold per tile, peaky (x4) rows, and rows whose maximum comes last — the model
must stay within the parity tolerances of the exact fp64 attention (O: the literal 1e-2
before the output rounding, 1e-2 plus half a bf16 ulp after it; LSE: 1e-3), and every
rounded P must stay finite and at most 2^8."""

import numpy as np
import pytest
import torch

LAZY, BN = 8.0, 128


def bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(
        torch.float32).numpy()


def model_row(x, v16):
    """x: log2-domain scores (fp32); v16: bf16-valued V (fp32 array).  Returns O before the
    output rounding (fp32), LSE and the largest rounded P."""
    m, l, lr = -np.inf, np.float32(0), np.float32(0)
    o = np.zeros(v16.shape[1], dtype=np.float32)
    pmax = 0.0
    for t0 in range(0, len(x), BN):
        xt = x[t0:t0 + BN]
        mt = np.float32(xt.max())
        if m == -np.inf or mt - m > LAZY:
            a = np.float32(0) if m == -np.inf else np.float32(np.exp2(np.float32(m - mt)))
            o, l, lr = o * a, np.float32(l * a), np.float32(lr * a)
            m = mt
        p = np.exp2((xt - m).astype(np.float32)).astype(np.float32)
        p16 = bf16(p)
        pmax = max(pmax, float(p16.max()))
        l = np.float32(l + p.sum(dtype=np.float32))
        lr = np.float32(lr + p16.sum(dtype=np.float32))
        o = (o + p16 @ v16[t0:t0 + BN]).astype(np.float32)
    lse = np.log(2.0) * (float(m) + np.log2(float(l)))
    return o / lr, lse, pmax


def exact_row(x, v16):
    x64 = x.astype(np.float64)
    w = np.exp2(x64 - x64.max())
    o = (w @ v16.astype(np.float64)) / w.sum()
    lse = np.log(2.0) * (x64.max() + np.log2(w.sum()))
    return o, lse


def rows(kind, n, rng):
    if kind == "climb":        # each tile's maximum 7.9 above the previous: no refresh
        return (np.arange(n) // BN * 7.9 + rng.standard_normal(n) * 0.1).astype(np.float32)
    if kind == "climb_fast":   # refreshes every tile
        return (np.arange(n) * 0.2 + rng.standard_normal(n)).astype(np.float32)
    if kind == "peaky":        # (4q)·(4k)/sqrt(d) with unit-normal q, k: std 16, in log2 units
        return (rng.standard_normal(n) * 16 * np.log2(np.e)).astype(np.float32)
    if kind == "max_last":
        x = rng.standard_normal(n).astype(np.float32)
        x[-1] = 40.0
        return x
    return rng.standard_normal(n).astype(np.float32) * np.float32(np.log2(np.e))


@pytest.mark.parametrize("kind", ["normal", "climb", "climb_fast", "peaky", "max_last"])
@pytest.mark.parametrize("n", [1, 129, 1000, 4096])
def test_model_within_parity_tolerance(kind, n):
    rng = np.random.default_rng(n + len(kind))
    for _ in range(4):
        x = rows(kind, n, rng)
        v16 = bf16(rng.standard_normal((n, 128)))
        o_pre, lse, pmax = model_row(x, v16)
        o_ref, lse_ref = exact_row(x, v16)
        # before the output rounding: the literal 1e-2
        assert np.all(np.abs(o_pre - o_ref) <= 1e-2), (kind, n, np.abs(o_pre - o_ref).max())
        # after rounding to bf16: 1e-2 plus half a bf16 ulp, as the GPU parity tests apply
        o = bf16(o_pre)
        half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(o_ref), 1e-30))) - 8)
        assert np.all(np.abs(o - o_ref) <= 1e-2 + half_ulp), (kind, n, np.abs(o - o_ref).max())
        assert abs(lse - lse_ref) <= 1e-3, (kind, n, lse - lse_ref)
        assert np.isfinite(pmax) and pmax <= 2.0 ** LAZY * (1 + 2 ** -8)
