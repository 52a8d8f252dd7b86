"""GPU parity of the FP8 forward (fa_fwd_fp8 / fa_varlen_fwd_fp8 through the C ABI)
against the oracle's attention of the dequantised E4M3 inputs.

Tolerance (derived from the arithmetic; the 1e-2 of the 16-bit path does not apply to
8-bit inputs).  The products are exact up to fp32 accumulation; the one 8-bit rounding
inside the kernel is of the softmax weights: p_j = 2^(x_j - m + 6), with m <= max x the
kernel's reference maximum, is rounded to E4M3 (relative error <= 2^-4 for normal values,
absolute <= 2^-10 below the normal range) and O = sum_j p~_j v_j / sum_j p~_j, whose
denominator is at least (1 - 2^-4) 2^6 sum_j 2^(x_j - max x).  Then, per element,

  |O_ic - O_ref,ic| <= 2^-4/(1 - 2^-4) * sum_j w_ij |v_jc - O_ref,ic|
                       + 2^-16/(1 - 2^-4) * sum_j |v_jc - O_ref,ic| / sum_j 2^(x_j - max x)
                       + 1e-3 (fp32 accumulation, exponential approximations)
                       + half a 16-bit ulp of O_ref (output rounding),

with w the exact softmax weights.  LSE comes from the unrounded weights: 1e-3 as for fa_fwd.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_33_b200 import attention as fa
from exact_tiled_attention_33_b200 import workloads as wl
from tests.parity import check_lse, f64, guard_intact, guarded_empty, half_ulp

pytestmark = pytest.mark.gpu
DEV = "cuda"
EPS8 = 2.0 ** -4


def u8(t):
    return t.view(torch.uint8).numpy()


def fp8_bound(q, k, v, scale, causal, rows, o_ref, dtype):
    """The per-element bound above for the listed rows (inputs dequantised, fp64)."""
    p = oracle.softmax_probs(q, k, scale, causal, rows=rows)          # exact weights w
    s = scale * (q[rows] @ k.T)
    mask = oracle.allowed_mask(np.asarray(rows), len(q), len(k), causal)
    s = np.where(mask, s, -np.inf)
    mx = np.max(s, axis=1, keepdims=True)
    rel = np.where(mask, np.exp(s - np.where(np.isfinite(mx), mx, 0.0)), 0.0)
    tot = np.maximum(rel.sum(axis=1), 1e-300)                          # sum_j 2^(x_j - max x)
    b1 = np.zeros_like(o_ref)
    b2 = np.zeros_like(o_ref)
    for i in range(len(rows)):                                         # one row at a time
        dev = np.abs(v - o_ref[i][None, :]) * mask[i][:, None]         # |v_j - O_i|, allowed j
        b1[i] = p[i] @ dev
        b2[i] = dev.sum(axis=0) / tot[i]
    return EPS8 / (1 - EPS8) * b1 + 2.0 ** -16 / (1 - EPS8) * b2 + 1e-3 + half_ulp(o_ref, dtype)


def check_fp8_o(o_gpu, o_ref, bound, what):
    err = np.abs(o_gpu - o_ref)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} over the bound; max err {err.max():.4g}"
    return float(err.max()), float((err / bound).max())


def run_dense(w, rows_per_head=None, pairs=None):
    t = wl.generate(w, with_grad_out=False)
    q8, k8, v8 = (t[x].to(DEV) for x in ("q8", "k8", "v8"))
    sq, sk, sv = t["q_descale"], t["k_descale"], t["v_descale"]
    B, N, H, d = q8.shape
    odt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    o, ob = guarded_empty((B, N, H, d), odt, DEV)
    lse, lb = guarded_empty((B, H, N), torch.float32, DEV)
    fa.fwd_fp8(q8, k8, v8, sq, sk, sv, w.softmax_scale, w.causal, out=o, lse=lse)
    assert fa.device_status() == 0
    assert guard_intact(ob, o.numel()) and guard_intact(lb, lse.numel())
    og, lg = f64(o), f64(lse)
    Q8, K8, V8 = (u8(t[x]) for x in ("q8", "k8", "v8"))
    worst = 0.0
    for (b, h) in (pairs or [(b, h) for b in range(B) for h in range(H)]):
        rows = np.arange(N) if rows_per_head is None else wl.sample_rows(N, rows_per_head, 7 + h)
        o_ref, l_ref = oracle.attention_forward_fp8(Q8[b, :, h], K8[b, :, h], V8[b, :, h], sq, sk,
                                                    sv, w.softmax_scale, w.causal, rows=rows)
        q = oracle.e4m3_to_float(Q8[b, :, h]) * sq
        k = oracle.e4m3_to_float(K8[b, :, h]) * sk
        v = oracle.e4m3_to_float(V8[b, :, h]) * sv
        bound = fp8_bound(q, k, v, w.softmax_scale, w.causal, rows, o_ref, w.dtype)
        _, ratio = check_fp8_o(og[b, rows, h], o_ref, bound, f"O[{b},{h}]")
        worst = max(worst, ratio)
        check_lse(lg[b, h, rows], l_ref, f"LSE[{b},{h}]")
    return o, lse, worst


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,H", [(1, 1, 1), (1, 2, 2), (2, 127, 2), (1, 129, 2), (1, 300, 2),
                                   (1, 1000, 1)])
def test_ragged_dense(B, N, H, causal):
    w = wl.custom("fp8_ragged", B=B, N=N, H=H, d=128, causal=causal, seed=60 + N, fp8=True)
    run_dense(w)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("scale", [0.0, 0.02, 0.3])
def test_scales_and_output_dtypes(dtype, scale):
    w = wl.custom("fp8_scales", B=1, N=400, H=2, d=128, dtype=dtype, causal=True, seed=61,
                  scale=scale, fp8=True)
    run_dense(w)


def test_peaky_inputs():
    # Q, K x4 before quantisation: nearly one-hot softmax rows, where the rounded weights'
    # normalisation by their own sum matters most
    w = wl.custom("fp8_peaky", B=1, N=700, H=2, d=128, causal=True, seed=62, qk_mult=4.0,
                  fp8=True)
    run_dense(w)


@pytest.mark.parametrize("name", ["fp8_long_causal", "fp8_long_noncausal"])
def test_long_sampled(name):
    run_dense(wl.get(name), rows_per_head=64, pairs=[(0, 0), (1, 31)])


def test_deterministic():
    w = wl.custom("fp8_det", B=1, N=600, H=2, d=128, causal=True, seed=63, fp8=True)
    o1, l1, _ = run_dense(w)
    o2, l2, _ = run_dense(w)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen(causal):
    lens_q = [1, 300, 0, 129, 77, 256, 513, 2]
    lens_k = [1, 300, 0, 200, 77, 100, 513, 9]
    cq = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    g = torch.Generator().manual_seed(64)
    H, d = 2, 128
    xs = [torch.randn((n, H, d), generator=g) for n in (cq[-1], ck[-1], ck[-1])]
    codes, descales = [], []
    for x in xs:
        ds = float(x.abs().max()) / 448.0
        codes.append((x / ds).to(torch.float8_e4m3fn))
        descales.append(ds)
    q8, k8, v8 = (c.to(DEV) for c in codes)
    cqd, ckd = torch.from_numpy(cq).to(DEV), torch.from_numpy(ck).to(DEV)
    o, lse = fa.varlen_fwd_fp8(q8, k8, v8, cqd, ckd, max(lens_q), max(lens_k), *descales,
                               softmax_scale=d ** -0.5, causal=causal)
    assert fa.device_status() == 0
    og, lg = f64(o), f64(lse)
    Q8, K8, V8 = (u8(c) for c in codes)
    for s in range(len(lens_q)):
        a, b, c0, c1 = cq[s], cq[s + 1], ck[s], ck[s + 1]
        if b == a:
            continue
        for h in range(H):
            rows = np.arange(b - a)
            o_ref, l_ref = oracle.attention_forward_fp8(Q8[a:b, h], K8[c0:c1, h], V8[c0:c1, h],
                                                        *descales, d ** -0.5, causal)
            if c1 == c0:
                assert np.all(og[a:b, h] == 0) and np.all(np.isposinf(lg[h, a:b]))
                continue
            q = oracle.e4m3_to_float(Q8[a:b, h]) * descales[0]
            k = oracle.e4m3_to_float(K8[c0:c1, h]) * descales[1]
            v = oracle.e4m3_to_float(V8[c0:c1, h]) * descales[2]
            bound = fp8_bound(q, k, v, d ** -0.5, causal, rows, o_ref, "bf16")
            check_fp8_o(og[a:b, h], o_ref, bound, f"varlen O seg {s} head {h}")
            check_lse(lg[h, a:b], l_ref, f"varlen LSE seg {s} head {h}")
