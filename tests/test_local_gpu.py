"""GPU parity of sliding-window (local) attention — fa_fwd_local, fa_varlen_fwd_local,
fa_bwd_local, fa_varlen_bwd_local through the C ABI — against the fp64 oracle's window
mask on seeded inputs, with the tolerances of the causal path (O 1e-2, LSE 1e-3,
gradients 2e-2 max|ref|).  Windows cover the degenerate one-key window, windows narrower
and wider than a 128-key tile, windows that end exactly on a tile boundary, asymmetric
and one-sided windows, Lq != Lk, empty windows and zero-length sequences."""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_33_b200 import attention as fa
from exact_tiled_attention_33_b200 import workloads as wl
from tests.parity import (check_grad, check_grad_segments, check_lse, check_o, f64, guard_intact,
                          guarded_empty, o16_term_in_d)

pytestmark = pytest.mark.gpu
DEV = "cuda"

WINDOWS = [(0, 0), (1, 0), (127, 0), (128, 0), (200, 0), (3, 5), (64, 64), (0, 130),
           (300, -1), (-1, 40)]


def dense_inputs(w):
    t = wl.generate(w)
    return t, tuple(t[x].to(DEV) for x in ("q", "k", "v", "do"))


def few_keys(window) -> bool:
    # rows see at most two keys: O is one value or the mix of two, |O| up to ~4
    wl_, wr_ = window
    return wl_ >= 0 and wr_ >= 0 and wl_ + wr_ <= 1


def run_fwd(w, rows_per_head=None, pairs=None):
    t, (q, k, v, _) = dense_inputs(w)
    B, N, H, d = q.shape
    o, ob = guarded_empty(q.shape, q.dtype, DEV)
    lse, lb = guarded_empty((B, H, N), torch.float32, DEV)
    fa.fwd_local(q, k, v, w.window, w.softmax_scale, out=o, lse=lse)
    assert fa.device_status() == 0
    assert guard_intact(ob, o.numel()) and guard_intact(lb, lse.numel())
    # the same kernel's fp32 output before rounding: held to the literal 1e-2 below, and the
    # 16-bit output is exactly it rounded
    o32, _ = fa.fwd_f32out(q, k, v, w.softmax_scale, window=w.window)
    assert fa.device_status() == 0
    assert torch.equal(o32.to(o.dtype), o)
    og, lg, og32 = f64(o), f64(lse), f64(o32)
    qf, kf, vf = (wl.to_f64(t[x]) for x in ("q", "k", "v"))
    for (b, h) in (pairs or [(b, h) for b in range(B) for h in range(H)]):
        rows = None if rows_per_head is None else wl.sample_rows(N, rows_per_head, 50 + b * H + h)
        o_ref, l_ref = oracle.attention_forward(qf[b, :, h], kf[b, :, h], vf[b, :, h],
                                                w.softmax_scale, False, rows=rows,
                                                window=w.window)
        sel = slice(None) if rows is None else rows
        check_o(og32[b, sel, h], o_ref, "fp32", f"O fp32[{b},{h}] window {w.window}")
        check_o(og[b, sel, h], o_ref, w.dtype, f"O[{b},{h}] window {w.window}",
                rounding_allowance=few_keys(w.window))
        check_lse(lg[b, h, sel], l_ref, f"LSE[{b},{h}] window {w.window}")
    return o, lse


def run_bwd(w, dq_rows=None, dkv_rows=None, pairs=None, deterministic=False):
    t, (q, k, v, do) = dense_inputs(w)
    B, N, H, d = q.shape
    o, lse = fa.fwd_local(q, k, v, w.window, w.softmax_scale)
    grads = [guarded_empty(q.shape, q.dtype, DEV) for _ in range(3)]
    (dq, gq), (dk, gk), (dv, gv) = grads
    fa.bwd_local(q, k, v, o, lse, do, w.window, w.softmax_scale, dq=dq, dk=dk, dv=dv,
                 deterministic=deterministic)
    assert fa.device_status() == 0
    assert all(guard_intact(g, q.numel()) for g in (gq, gk, gv))
    dqg, dkg, dvg = f64(dq), f64(dk), f64(dv)
    qf, kf, vf, dof = (wl.to_f64(t[x]) for x in ("q", "k", "v", "do"))
    degenerate = tuple(w.window) == (0, 0)  # one key per row: exact dQ = dK = 0
    for (b, h) in (pairs or [(b, h) for b in range(B) for h in range(H)]):
        qr = None if dq_rows is None else wl.sample_rows(N, dq_rows, 70 + b * H + h)
        kr = None if dkv_rows is None else wl.sample_rows(N, dkv_rows, 90 + b * H + h)
        args = (qf[b, :, h], kf[b, :, h], vf[b, :, h], dof[b, :, h], w.softmax_scale, False)
        gq_ref, _, _ = oracle.attention_backward(*args, dq_rows=qr,
                                                 dkv_rows=np.zeros(0, np.int64), window=w.window)
        _, gk_ref, gv_ref = oracle.attention_backward(*args, dq_rows=np.zeros(0, np.int64),
                                                      dkv_rows=kr, window=w.window)
        eq = ek = None
        if degenerate:
            bq, bk = o16_term_in_d(*args[:5], False, w.dtype, window=w.window)
            eq = bq if qr is None else bq[qr]
            ek = bk if kr is None else bk[kr]
        sq = slice(None) if qr is None else qr
        sk = slice(None) if kr is None else kr
        tag = f"[{b},{h}] window {w.window}"
        check_grad(dqg[b, sq, h], gq_ref, "dQ" + tag, extra=eq)
        check_grad(dkg[b, sk, h], gk_ref, "dK" + tag, extra=ek)
        check_grad(dvg[b, sk, h], gv_ref, "dV" + tag)
    return dq, dk, dv


# ------------------------------------------------------------------ dense forward
@pytest.mark.parametrize("window", WINDOWS)
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [300, 1000])
def test_fwd_windows(N, d, window):
    w = wl.custom("local_fwd", B=1, N=N, H=2, d=d, seed=100 + N + d, window=window)
    run_fwd(w)


@pytest.mark.parametrize("window", [(0, 0), (1, 0), (5, 5), (-1, 3), (2, -1)])
@pytest.mark.parametrize("N", [1, 2, 129])
def test_fwd_small_sizes(N, window):
    w = wl.custom("local_small", B=2, N=N, H=2, d=128, seed=7 + N, window=window)
    run_fwd(w)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("scale", [0.0, -0.3])
def test_fwd_scales_and_dtypes(dtype, scale):
    w = wl.custom("local_scales", B=1, N=400, H=2, d=64, dtype=dtype, seed=9, scale=scale,
                  window=(100, 20))
    run_fwd(w)


def test_window_matches_causal_and_full_bitwise():
    # (-1, 0) is the causal mask and (-1, -1) / bounds beyond the sequence are full
    # attention: the same kernels run the same tiles, so results agree bit for bit.
    w = wl.custom("local_eq", B=2, N=700, H=2, d=128, seed=11)
    t, (q, k, v, do) = dense_inputs(w)
    oc, lc = fa.fwd(q, k, v, None, True)
    on, ln = fa.fwd(q, k, v, None, False)
    for win, (o_ref, l_ref) in (((-1, 0), (oc, lc)), ((700, 0), (oc, lc)),
                                ((-1, -1), (on, ln)), ((699, 699), (on, ln)),
                                ((5000, 5000), (on, ln))):
        o, l = fa.fwd_local(q, k, v, win)
        assert torch.equal(o, o_ref) and torch.equal(l, l_ref), win
    gc = fa.bwd(q, k, v, oc, lc, do, None, True, deterministic=True)
    gl = fa.bwd_local(q, k, v, oc, lc, do, (-1, 0), deterministic=True)
    assert all(torch.equal(a, b) for a, b in zip(gc, gl))
    # single pass: dK and dV are written once per key tile, so they agree bitwise too
    gc = fa.bwd(q, k, v, oc, lc, do, None, True)
    gl = fa.bwd_local(q, k, v, oc, lc, do, (-1, 0))
    assert torch.equal(gc[1], gl[1]) and torch.equal(gc[2], gl[2])
    assert fa.device_status() == 0


def test_long_local_sampled():
    w = wl.get("long_local_w4096")
    run_fwd(w, rows_per_head=128, pairs=[(0, 0), (0, 17), (1, 5), (1, 31)])


def test_long_local_symmetric_sampled():
    w = wl.get("long_local_sym512")
    run_fwd(w, rows_per_head=128, pairs=[(0, 3), (1, 30)])


# ------------------------------------------------------------------ dense backward
@pytest.mark.parametrize("deterministic", [False, True])
@pytest.mark.parametrize("window", [(0, 0), (1, 0), (127, 0), (128, 0), (3, 5), (64, 64),
                                    (0, 130), (300, -1), (-1, 40)])
@pytest.mark.parametrize("d", [64, 128])
def test_bwd_windows(d, window, deterministic):
    w = wl.custom("local_bwd", B=1, N=520, H=2, d=d, seed=200 + d, window=window)
    run_bwd(w, deterministic=deterministic)


def test_bwd_long_local_sampled():
    w = wl.get("long_local_w4096")
    run_bwd(w, dq_rows=64, dkv_rows=64, pairs=[(0, 1), (1, 20)])


def test_bwd_deterministic():
    w = wl.custom("local_det", B=1, N=600, H=2, d=128, seed=12, window=(150, 30))
    g1 = run_bwd(w, deterministic=True)
    g2 = run_bwd(w, deterministic=True)
    assert all(torch.equal(a, b) for a, b in zip(g1, g2))


def test_autograd_window():
    w = wl.custom("local_autograd", B=1, N=300, H=2, d=64, seed=13, window=(40, 0))
    t, (q, k, v, do) = dense_inputs(w)
    qq, kk, vv = (x.clone().requires_grad_(True) for x in (q, k, v))
    out = fa.flash_attn_func(qq, kk, vv, None, False, window=(40, 0), deterministic=True)
    out.backward(do)
    o, lse = fa.fwd_local(q, k, v, (40, 0))
    dq, dk, dv = fa.bwd_local(q, k, v, o, lse, do, (40, 0), deterministic=True)
    assert torch.equal(out.detach(), o)
    assert torch.equal(qq.grad, dq) and torch.equal(kk.grad, dk) and torch.equal(vv.grad, dv)


# ------------------------------------------------------------------ varlen
def run_varlen(lens_q, lens_k, H, d, window, seed, bwd=True):
    cq = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    g = torch.Generator().manual_seed(seed)
    tq, tk = int(cq[-1]), int(ck[-1])
    q = torch.randn((tq, H, d), generator=g).to(torch.bfloat16)
    k = torch.randn((tk, H, d), generator=g).to(torch.bfloat16)
    v = torch.randn((tk, H, d), generator=g).to(torch.bfloat16)
    do = torch.randn((tq, H, d), generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = (x.to(DEV) for x in (q, k, v, do))
    cqd, ckd = torch.from_numpy(cq).to(DEV), torch.from_numpy(ck).to(DEV)
    mq, mk = max(lens_q), max(lens_k)
    scale = d ** -0.5
    o, lse = fa.varlen_fwd_local(qd, kd, vd, cqd, ckd, mq, mk, window, scale)
    assert fa.device_status() == 0
    qf, kf, vf, dof = (wl.to_f64(x) for x in (q, k, v, do))
    o_ref, l_ref = oracle.varlen_attention_forward(qf, kf, vf, cq, ck, scale, False,
                                                   window=window)
    check_o(f64(o), o_ref, "bf16", f"varlen O window {window}")
    check_lse(f64(lse), l_ref, f"varlen LSE window {window}")
    if not bwd:
        return
    dq, dk, dv = fa.varlen_bwd_local(qd, kd, vd, o, lse, dod, cqd, ckd, mq, mk, window, scale)
    assert fa.device_status() == 0
    gq, gk, gv = oracle.varlen_attention_backward(qf, kf, vf, dof, cq, ck, scale, False,
                                                  window=window)
    # per (segment, head) scale; a window of one key per row makes the exact dQ = dK = 0
    check_grad_segments([f64(dq), f64(dk), f64(dv)], (gq, gk, gv), cq, ck,
                        f"varlen window {window}", scale, False, "bf16", qf, kf, vf, dof,
                        window=window)


@pytest.mark.parametrize("window", [(1, 0), (100, 0), (128, 3), (20, 20), (-1, 7), (50, -1)])
def test_varlen_windows(window):
    lens = [1, 300, 0, 129, 77, 256, 513, 2]
    run_varlen(lens, lens, 2, 128, window, seed=21)


@pytest.mark.parametrize("window", [(0, 0), (30, 0), (10, 10), (200, 5)])
def test_varlen_unequal_q_k(window):
    # Lq != Lk per sequence: the window sits on the bottom-right diagonal; with Lq > Lk
    # and a short window, early rows see no key at all.
    lens_q = [10, 290, 5, 130, 1, 300]
    lens_k = [50, 50, 0, 400, 7, 140]
    run_varlen(lens_q, lens_k, 2, 64, window, seed=22)
