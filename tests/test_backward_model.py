"""CPU model of the backward passes' arithmetic as built (not of their code): P recomputed in
fp32 from the scores and the forward's LSE, rounded to bf16 before it enters a product;
D = rowsum(dO ∘ O) from the bf16 O the caller passes; dS = P̃ ∘ (dP − D) rounded to bf16;
every product accumulated in fp32 from bf16 operands.  On normal and peaky (Q, K x4) inputs,
causal and not, the model's dQ, dK, dV must stay within the parity tolerance
(2e-2 · max|ref|) of the oracle's fp64 gradients — the same check the GPU tests apply."""

import numpy as np
import pytest
import torch

import oracle


def bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(
        torch.float32).numpy()


def f32_matmul(a, b):
    return (a.astype(np.float32) @ b.astype(np.float32)).astype(np.float32)


def model_backward(q, k, v, do, o16, lse, scale, causal):
    n = q.shape[0]
    s = f32_matmul(q, k.T)
    x = (s * np.float32(scale * np.log2(np.e)) - (lse * np.log2(np.e))[:, None]).astype(np.float32)
    if causal:   # masked pairs give exactly 0 (the kernels select 0 for them)
        x = np.where(np.tril(np.ones((n, n), bool)), x, np.float32(-np.inf))
    p = np.exp2(x).astype(np.float32)
    p16 = bf16(p)
    dmat = (do.astype(np.float32) * o16.astype(np.float32)).sum(axis=1, dtype=np.float32)
    dp = f32_matmul(do, v.T)
    ds16 = bf16(p16 * (dp - dmat[:, None]))
    dv = f32_matmul(p16.T, do)
    dk = (np.float32(scale) * f32_matmul(ds16.T, q)).astype(np.float32)
    dq = (np.float32(scale) * f32_matmul(ds16, k)).astype(np.float32)
    return bf16(dq), bf16(dk), bf16(dv)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("mult", [1.0, 4.0])
@pytest.mark.parametrize("n", [128, 700])
def test_model_gradients_within_tolerance(causal, mult, n):
    rng = np.random.default_rng(int(n + 10 * mult + causal))
    d = 128
    scale = d ** -0.5
    q, k = (bf16(rng.standard_normal((n, d)) * mult) for _ in range(2))
    v, do = (bf16(rng.standard_normal((n, d))) for _ in range(2))
    q64, k64, v64, do64 = (a.astype(np.float64) for a in (q, k, v, do))
    o_ref, lse_ref = oracle.attention_forward(q64, k64, v64, scale, causal)
    o16 = bf16(o_ref)                                   # the forward's stored output
    lse = lse_ref.astype(np.float32)                    # the forward's stored LSE (fp32)
    dq, dk, dv = model_backward(q, k, v, do, o16, lse, scale, causal)
    refs = oracle.attention_backward(q64, k64, v64, do64, scale, causal)
    for name, g, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), refs):
        err = np.abs(g - r).max()
        assert err <= 2e-2 * np.abs(r).max(), (name, causal, mult, n, err / np.abs(r).max())
