"""GPU parity of the backward pass (fa_bwd / fa_varlen_bwd through the C ABI) against the
fp64 oracle's analytic gradients on seeded inputs: max |dX - dX_ref| <= 2e-2 max |dX_ref|
for dX in dQ, dK, dV.  The forward outputs (O, LSE) fed to the backward pass come from
the library's own forward kernel, as in training."""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_33_b200 import attention as fa
from exact_tiled_attention_33_b200 import workloads as wl
from tests.parity import (check_grad, check_grad_segments, f64, guard_intact, guarded_empty,
                          o16_term_in_d)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_dense_bwd(w, dq_rows=None, dkv_rows=None, dkv_heads=None, dq_heads=None,
                  d16_term=False, deterministic=False):
    t = wl.generate(w)
    q, k, v, do = (t[x].to(DEV) for x in ("q", "k", "v", "do"))
    B, N, H, d = q.shape
    o, lse = fa.fwd(q, k, v, w.softmax_scale, w.causal)
    dq, gq = guarded_empty(q.shape, q.dtype, DEV)
    dk, gk = guarded_empty(q.shape, q.dtype, DEV)
    dv, gv = guarded_empty(q.shape, q.dtype, DEV)
    fa.bwd(q, k, v, o, lse, do, w.softmax_scale, w.causal, dq=dq, dk=dk, dv=dv,
           deterministic=deterministic)
    assert fa.device_status() == 0
    n = q.numel()
    assert guard_intact(gq, n) and guard_intact(gk, n) and guard_intact(gv, n)
    dqg, dkg, dvg = f64(dq), f64(dk), f64(dv)
    qf, kf, vf, dof = (wl.to_f64(t[x]) for x in ("q", "k", "v", "do"))
    all_pairs = [(b, h) for b in range(B) for h in range(H)]
    errs = {"dq": 0.0, "dk": 0.0, "dv": 0.0}
    # dQ on sampled query rows of every listed (b, h)
    for (b, h) in (all_pairs if dq_heads is None else dq_heads):
        rows = None if dq_rows is None else wl.sample_rows(N, dq_rows, 3000 + b * H + h)
        gq_ref, _, _ = oracle.attention_backward(qf[b, :, h], kf[b, :, h], vf[b, :, h],
                                                 dof[b, :, h], w.softmax_scale, w.causal,
                                                 dq_rows=rows, dkv_rows=np.zeros(0, np.int64))
        sel = slice(None) if rows is None else rows
        extra = None
        if d16_term:
            extra = o16_term_in_d(qf[b, :, h], kf[b, :, h], vf[b, :, h], dof[b, :, h],
                                  w.softmax_scale, w.causal, w.dtype)[0][sel]
        errs["dq"] = max(errs["dq"], check_grad(dqg[b, sel, h], gq_ref, f"dQ[{b},{h}]",
                                                extra=extra))
    # dK, dV on sampled key rows of the listed (b, h)
    for (b, h) in (all_pairs if dkv_heads is None else dkv_heads):
        rows = None if dkv_rows is None else wl.sample_rows(N, dkv_rows, 4000 + b * H + h)
        _, gk_ref, gv_ref = oracle.attention_backward(qf[b, :, h], kf[b, :, h], vf[b, :, h],
                                                      dof[b, :, h], w.softmax_scale, w.causal,
                                                      dq_rows=np.zeros(0, np.int64), dkv_rows=rows)
        sel = slice(None) if rows is None else rows
        extra = None
        if d16_term:
            extra = o16_term_in_d(qf[b, :, h], kf[b, :, h], vf[b, :, h], dof[b, :, h],
                                  w.softmax_scale, w.causal, w.dtype)[1][sel]
        errs["dk"] = max(errs["dk"], check_grad(dkg[b, sel, h], gk_ref, f"dK[{b},{h}]",
                                                extra=extra))
        errs["dv"] = max(errs["dv"], check_grad(dvg[b, sel, h], gv_ref, f"dV[{b},{h}]"))
    return errs, (dq, dk, dv)


@pytest.mark.parametrize("name", ["tiny_noncausal", "tiny_causal"])
def test_tiny(name):
    run_dense_bwd(wl.get(name))


@pytest.mark.parametrize("deterministic", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,H", [(1, 1, 1), (1, 2, 2), (2, 127, 2), (1, 129, 2), (1, 300, 2),
                                   (1, 513, 1)])
def test_ragged_dense(B, N, H, d, causal, deterministic):
    w = wl.custom("bwd_ragged", B=B, N=N, H=H, d=d, causal=causal, seed=41 + N)
    run_dense_bwd(w, d16_term=N <= 2, deterministic=deterministic)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("scale", [0.0, -0.25, 0.05])
def test_scales_and_dtypes(dtype, scale):
    w = wl.custom("bwd_scales", B=1, N=260, H=2, d=128, dtype=dtype, causal=True, seed=6,
                  scale=scale)
    run_dense_bwd(w)


def test_a100_table_n1024_full():
    run_dense_bwd(wl.get("a100table_N1024"))


@pytest.mark.parametrize("name", ["a100table_N2048", "a100table_N4096"])
def test_a100_table_sampled(name):
    run_dense_bwd(wl.get(name), dq_rows=256, dkv_rows=256, dkv_heads=[(0, 0), (3, 7), (5, 12),
                                                                      (7, 15)])


@pytest.mark.parametrize("name", ["llama_causal", "llama_noncausal"])
def test_llama_sampled(name):
    run_dense_bwd(wl.get(name), dq_rows=256, dkv_rows=256,
                  dkv_heads=[(0, 0), (1, 17), (2, 5), (3, 31)])


@pytest.mark.parametrize("name", ["long_causal", "long_noncausal", "long_peaky_causal",
                                  "long_peaky_noncausal"])
def test_long_sampled(name):
    run_dense_bwd(wl.get(name), dq_rows=128, dkv_rows=128, dkv_heads=[(0, 3), (1, 30)],
                  dq_heads=[(0, h) for h in range(0, 32, 4)] + [(1, h) for h in range(1, 32, 4)])


@pytest.mark.parametrize("name", ["long_causal", "long_peaky_noncausal"])
def test_long_sampled_deterministic(name):
    run_dense_bwd(wl.get(name), dq_rows=128, dkv_rows=128, dkv_heads=[(0, 3), (1, 30)],
                  dq_heads=[(0, 0), (1, 31)], deterministic=True)


def test_deterministic():
    # deterministic mode: every gradient element is written exactly once (no atomics), so
    # dQ, dK and dV are bitwise reproducible
    w = wl.custom("bwd_det", B=1, N=600, H=2, d=128, causal=True, seed=8)
    _, (dq1, dk1, dv1) = run_dense_bwd(w, deterministic=True)
    _, (dq2, dk2, dv2) = run_dense_bwd(w, deterministic=True)
    assert torch.equal(dq1, dq2) and torch.equal(dk1, dk2) and torch.equal(dv1, dv2)


@pytest.mark.parametrize("causal", [False, True])
def test_single_pass_dk_dv_reproducible(causal):
    # the single-pass backward writes dK and dV once per key tile (bitwise reproducible); dQ
    # is a sum of atomic fp32 adds whose order varies, so it is checked against the oracle
    # (run_dense_bwd) and against the deterministic mode within the gradient tolerance
    w = wl.custom("bwd_sp_det", B=2, N=900, H=3, d=128, causal=causal, seed=18)
    _, (dq1, dk1, dv1) = run_dense_bwd(w)
    _, (dq2, dk2, dv2) = run_dense_bwd(w)
    _, (dq3, _, _) = run_dense_bwd(w, deterministic=True)
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    for a in (dq2, dq3):
        check_grad(f64(dq1), f64(a), "dQ single pass vs repeat / deterministic")


def test_autograd_sum_loss():
    # loss = output.sum(); loss.backward(): gradients have the inputs' shapes, and with
    # dO = 1 the oracle's dV is the column sums of P.
    w = wl.custom("autograd", B=2, N=384, H=4, d=64, causal=True, seed=21)
    t = wl.generate(w, with_grad_out=False)
    q, k, v = (t[x].to(DEV).requires_grad_(True) for x in ("q", "k", "v"))
    o = fa.flash_attn_func(q, k, v, w.softmax_scale, True)
    o.float().sum().backward()
    assert q.grad.shape == q.shape and k.grad.shape == k.shape and v.grad.shape == v.shape
    qf, kf, vf = (wl.to_f64(t[x]) for x in ("q", "k", "v"))
    for (b, h) in [(0, 0), (1, 3)]:
        ones = np.ones((w.N, w.d))
        gq, gk, gv = oracle.attention_backward(qf[b, :, h], kf[b, :, h], vf[b, :, h], ones,
                                               w.softmax_scale, True)
        check_grad(f64(q.grad)[b, :, h], gq, "dQ")
        check_grad(f64(k.grad)[b, :, h], gk, "dK")
        check_grad(f64(v.grad)[b, :, h], gv, "dV")


# ------------------------------------------------------------------------------ varlen
def run_varlen_bwd(lens_q, lens_k, H, d, causal, dtype="bf16", seed=3, perturb=None,
                   deterministic=False, nan_fill=False):
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    w = wl.custom("varlen_bwd", seqlens=lens_q, H=H, d=d, dtype=dtype, causal=causal, seed=seed)
    g = torch.Generator().manual_seed(seed)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    q = torch.randn((tq, H, d), generator=g).to(w.torch_dtype)
    k = torch.randn((tk, H, d), generator=g).to(w.torch_dtype)
    v = torch.randn((tk, H, d), generator=g).to(w.torch_dtype)
    do = torch.randn((tq, H, d), generator=g).to(w.torch_dtype)
    if perturb is not None:
        q, k, v, do = perturb(q, k, v, do, cu_q, cu_k)
    qd, kd, vd, dod = (x.to(DEV) for x in (q, k, v, do))
    cq, ck = torch.from_numpy(cu_q).to(DEV), torch.from_numpy(cu_k).to(DEV)
    mq, mk = max(lens_q), max(lens_k)
    o, lse = fa.varlen_fwd(qd, kd, vd, cq, ck, mq, mk, w.softmax_scale, causal)
    # nan_fill: gradients start as NaN, so a key tile that no CTA covers cannot pass
    pre = ([torch.full_like(x, float("nan")) for x in (qd, kd, vd)] if nan_fill
           else [None, None, None])
    dq, dk, dv = fa.varlen_bwd(qd, kd, vd, o, lse, dod, cq, ck, mq, mk, w.softmax_scale, causal,
                               deterministic=deterministic, dq=pre[0], dk=pre[1], dv=pre[2])
    assert fa.device_status() == 0
    qf, kf, vf, dof = (wl.to_f64(x) for x in (q, k, v, do))
    ref = oracle.varlen_attention_backward(qf, kf, vf, dof, cu_q, cu_k, w.softmax_scale, causal)
    got = [f64(x) for x in (dq, dk, dv)]
    check_grad_segments(got, ref, cu_q, cu_k, "varlen", w.softmax_scale, causal, dtype,
                        qf, kf, vf, dof)
    return dq, dk, dv, cu_q, cu_k


def test_varlen_pages_example():
    w = wl.get("varlen3")
    run_varlen_bwd(list(w.seqlens), list(w.seqlens), w.H, w.d, True)


@pytest.mark.parametrize("deterministic", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_ragged(d, causal, deterministic):
    lens = [1, 300, 0, 129, 77, 256, 2]
    run_varlen_bwd(lens, lens, 2, d, causal, seed=14, deterministic=deterministic)


def _many_lengths(n, hi, long_len, seed):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, hi + 1, size=n).tolist()
    lens[n // 3] = long_len
    return lens


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_many_segments_packed_grid(causal):
    # 200 segments (lengths 0..100, one of 1000, some empty): the single-pass kernel's packed
    # grid over key tiles, found by a seven-step prefix sum over cu_seqlens_k
    lens = _many_lengths(200, 100, 1000, 43)
    run_varlen_bwd(lens, lens, 2, 64, causal, seed=43, nan_fill=True)


def test_varlen_over_1024_segments_per_segment_grid():
    lens = _many_lengths(1100, 40, 300, 44)
    run_varlen_bwd(lens, lens, 2, 64, True, seed=44, nan_fill=True)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_unequal_q_k(causal):
    run_varlen_bwd([10, 290, 5, 130, 1], [50, 50, 7, 400, 7], 2, 128, causal, seed=15)


@pytest.mark.parametrize("deterministic", [False, True])
def test_varlen_segment_isolation(deterministic):
    lens = [100, 200, 150]

    def bump(q, k, v, do, cu_q, cu_k):
        # other segments change (scaled, sign-flipped); the middle one does not
        q, k, v, do = (x.clone() for x in (q, k, v, do))
        for x in (q, k, v, do):
            x[cu_q[0]:cu_q[1]] = (x[cu_q[0]:cu_q[1]].float() * 0.5).to(x.dtype)
            x[cu_q[2]:cu_q[3]] = (-x[cu_q[2]:cu_q[3]].float()).to(x.dtype)
        return q, k, v, do

    dq1, dk1, dv1, cu, _ = run_varlen_bwd(lens, lens, 2, 64, True, seed=16,
                                          deterministic=deterministic)
    dq2, dk2, dv2, _, _ = run_varlen_bwd(lens, lens, 2, 64, True, seed=16, perturb=bump,
                                         deterministic=deterministic)
    a, b = cu[1], cu[2]
    # the untouched middle segment's dK and dV are bit-identical
    assert torch.equal(dk1[a:b], dk2[a:b]) and torch.equal(dv1[a:b], dv2[a:b])
    if deterministic:
        assert torch.equal(dq1[a:b], dq2[a:b])
    else:
        # its dQ sums only the segment's own key tiles (other segments add exactly nothing),
        # in an order that may vary: within the gradient tolerance of the first run
        check_grad(f64(dq2[a:b]), f64(dq1[a:b]), "isolated segment dQ")


def test_varlen64_sampled():
    w = wl.get("varlen64")
    t = wl.generate(w)
    cu = t["cu_seqlens"].numpy()
    q, k, v, do = (t[x].to(DEV) for x in ("q", "k", "v", "do"))
    cud = t["cu_seqlens"].to(DEV)
    L = max(w.seqlens)
    o, lse = fa.varlen_fwd(q, k, v, cud, cud, L, L, w.softmax_scale, True)
    dq, dk, dv = fa.varlen_bwd(q, k, v, o, lse, do, cud, cud, L, L, w.softmax_scale, True)
    assert fa.device_status() == 0
    dqg, dkg, dvg = f64(dq), f64(dk), f64(dv)
    qf, kf, vf, dof = (wl.to_f64(t[x]) for x in ("q", "k", "v", "do"))
    rng = np.random.default_rng(44)
    for s in rng.choice(64, size=4, replace=False):
        a, b = int(cu[s]), int(cu[s + 1])
        rows = wl.sample_rows(b - a, 64, 5000 + int(s))
        for h in rng.choice(w.H, size=2, replace=False):
            gq, gk, gv = oracle.attention_backward(qf[a:b, h], kf[a:b, h], vf[a:b, h], dof[a:b, h],
                                                   w.softmax_scale, True, dq_rows=rows,
                                                   dkv_rows=rows)
            check_grad(dqg[a + rows, h], gq, "dQ")
            check_grad(dkg[a + rows, h], gk, "dK")
            check_grad(dvg[a + rows, h], gv, "dV")
