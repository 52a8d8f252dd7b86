"""GPU parity of the forward pass (fa_fwd / fa_varlen_fwd through the C ABI) against the
fp64 CPU oracle on seeded inputs.  Sizes span several 128-row tiles with ragged tails;
edge cases cover N = 1, a single key, fully masked rows, zero-length sequences, Lq != Lk
and unusual scales.  Outputs are NaN-prefilled and followed by guard regions."""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_33_b200 import attention as fa
from exact_tiled_attention_33_b200 import workloads as wl
from tests.parity import check_lse, check_o, f64, guard_intact, guarded_empty

pytestmark = pytest.mark.gpu

DEV = "cuda"


def is_peaky(w) -> bool:
    # the Q,K x4 workloads: the only ones whose stored O may add half a 16-bit ulp
    return getattr(w, "qk_mult", 1.0) != 1.0


def run_dense(w, rows_per_head=None, bh_subset=None):
    t = wl.generate(w, with_grad_out=False)
    q, k, v = (t[x].to(DEV) for x in ("q", "k", "v"))
    B, N, H, d = q.shape
    o, obuf = guarded_empty((B, N, H, d), q.dtype, DEV)
    lse, lbuf = guarded_empty((B, H, N), torch.float32, DEV)
    fa.fwd(q, k, v, w.softmax_scale, w.causal, out=o, lse=lse)
    assert fa.device_status() == 0
    assert guard_intact(obuf, o.numel()) and guard_intact(lbuf, lse.numel())
    og, lg = f64(o), f64(lse)
    qf, kf, vf = (wl.to_f64(t[x]) for x in ("q", "k", "v"))
    pairs = [(b, h) for b in range(B) for h in range(H)] if bh_subset is None else bh_subset
    eo = el = 0.0
    for (b, h) in pairs:
        rows = None if rows_per_head is None else wl.sample_rows(N, rows_per_head, 1000 + b * H + h)
        o_ref, lse_ref = oracle.attention_forward(qf[b, :, h], kf[b, :, h], vf[b, :, h],
                                                  w.softmax_scale, w.causal, rows=rows)
        sel = slice(None) if rows is None else rows
        eo = max(eo, check_o(og[b, sel, h], o_ref, w.dtype, f"O[b={b},h={h}]",
                             rounding_allowance=is_peaky(w)))
        el = max(el, check_lse(lg[b, h, sel], lse_ref, f"LSE[b={b},h={h}]"))
    return eo, el, o, lse


@pytest.mark.parametrize("name", ["tiny_noncausal", "tiny_causal"])
def test_tiny(name):
    run_dense(wl.get(name))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,H", [(1, 1, 1), (1, 2, 2), (2, 127, 3), (1, 129, 2), (1, 255, 1),
                                   (1, 257, 2), (2, 300, 2), (1, 513, 1), (1, 1000, 1)])
def test_ragged_dense(B, N, H, d, causal):
    w = wl.custom(f"ragged_{B}_{N}_{H}_{d}_{causal}", B=B, N=N, H=H, d=d, causal=causal,
                  seed=17 + N)
    run_dense(w)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("scale", [0.0, -0.3, 0.02, 1.0])
def test_scales_and_dtypes(dtype, scale):
    w = wl.custom("scales", B=1, N=300, H=2, d=64, dtype=dtype, causal=True, seed=5, scale=scale)
    run_dense(w)


def test_a100_table_n1024_all_rows():
    run_dense(wl.get("a100table_N1024"))


@pytest.mark.parametrize("name", ["a100table_N2048", "a100table_N4096"])
def test_a100_table_sampled(name):
    run_dense(wl.get(name), rows_per_head=256)


@pytest.mark.parametrize("name", ["llama_causal", "llama_noncausal"])
def test_llama_sampled(name):
    w = wl.get(name)
    run_dense(w, rows_per_head=256)


@pytest.mark.parametrize("name", ["long_causal", "long_noncausal", "long_peaky_causal",
                                  "long_peaky_noncausal"])
def test_long_sampled(name):
    w = wl.get(name)
    run_dense(w, rows_per_head=128)


@pytest.mark.parametrize("name", ["long_peaky_causal", "long_peaky_noncausal"])
def test_long_peaky_fp32_output_literal_bound(name):
    # The same kernel with O written in fp32 before rounding: the literal |O - O_ref| <= 1e-2
    # holds on the peaky workloads too, where only the 16-bit rounding of |O| ~ 5 can exceed it.
    w = wl.get(name)
    t = wl.generate(w, with_grad_out=False)
    q, k, v = (t[x].to(DEV) for x in ("q", "k", "v"))
    o32, lse = fa.fwd_f32out(q, k, v, w.softmax_scale, w.causal)
    o16, lse16 = fa.fwd(q, k, v, w.softmax_scale, w.causal)
    assert fa.device_status() == 0
    # the 16-bit entry point returns exactly this fp32 output rounded to nearest-even
    assert torch.equal(o32.to(o16.dtype), o16) and torch.equal(lse, lse16)
    og, lg = f64(o32), f64(lse)
    qf, kf, vf = (wl.to_f64(t[x]) for x in ("q", "k", "v"))
    B, N, H, _ = q.shape
    for b in range(B):
        for h in range(0, H, 3):
            rows = wl.sample_rows(N, 128, 1000 + b * H + h)
            o_ref, lse_ref = oracle.attention_forward(qf[b, :, h], kf[b, :, h], vf[b, :, h],
                                                      w.softmax_scale, w.causal, rows=rows)
            check_o(og[b, rows, h], o_ref, "fp32", f"O fp32[b={b},h={h}]")
            check_lse(lg[b, h, rows], lse_ref, f"LSE[b={b},h={h}]")


def test_deterministic():
    w = wl.custom("det", B=2, N=700, H=3, d=128, causal=True, seed=9)
    _, _, o1, l1 = run_dense(w)
    _, _, o2, l2 = run_dense(w)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_page_shape_example():
    # q, k, v of shape (4, 4096, 32, 128) fp16 causal -> output (4, 4096, 32, 128).
    w = wl.get("llama_causal")
    t = wl.generate(w, with_grad_out=False)
    q, k, v = (t[x].to(DEV) for x in ("q", "k", "v"))
    o = fa.flash_attn_func(q, k, v, None, True)
    assert list(o.shape) == [4, 4096, 32, 128]


# ------------------------------------------------------------------------------ varlen
def run_varlen(lens_q, lens_k, H, d, causal, dtype="bf16", seed=3, scale=None, perturb=None):
    w = wl.custom("varlen", seqlens=lens_q, H=H, d=d, dtype=dtype, causal=causal, seed=seed,
                  scale=scale)
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    g = torch.Generator().manual_seed(seed)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    q = torch.randn((tq, H, d), generator=g).to(w.torch_dtype)
    k = torch.randn((tk, H, d), generator=g).to(w.torch_dtype)
    v = torch.randn((tk, H, d), generator=g).to(w.torch_dtype)
    if perturb is not None:
        k, v = perturb(k, v, cu_k)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    cq, ck = torch.from_numpy(cu_q).to(DEV), torch.from_numpy(cu_k).to(DEV)
    o, obuf = guarded_empty((tq, H, d), qd.dtype, DEV)
    lse, lbuf = guarded_empty((H, tq), torch.float32, DEV)
    fa.varlen_fwd(qd, kd, vd, cq, ck, max(lens_q), max(lens_k), w.softmax_scale, causal,
                  out=o, lse=lse)
    assert fa.device_status() == 0
    assert guard_intact(obuf, o.numel()) and guard_intact(lbuf, lse.numel())
    o_ref, lse_ref = oracle.varlen_attention_forward(wl.to_f64(q), wl.to_f64(k), wl.to_f64(v),
                                                     cu_q, cu_k, w.softmax_scale, causal)
    # the perturbed inputs of the isolation test shift one segment's V by -2 (|O| ~ 2, where
    # half a bf16 ulp is 2^-8): the stored output gets the output-rounding allowance there
    check_o(f64(o), o_ref, dtype, rounding_allowance=perturb is not None)
    check_lse(f64(lse), lse_ref)
    return o, lse, cu_q


def test_varlen_pages_example():
    # Three sequences of lengths 128/256/512, cu_seqlens [0,128,384,896], causal.
    w = wl.get("varlen3")
    o, _, cu = run_varlen(list(w.seqlens), list(w.seqlens), w.H, w.d, True)
    assert cu.tolist() == [0, 128, 384, 896] and list(o.shape) == [896, 32, 128]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_ragged(d, causal):
    lens = [1, 300, 0, 129, 77, 256, 513, 2]
    run_varlen(lens, lens, 3, d, causal, seed=11)


def _many_lengths(n, hi, long_len, seed):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, hi + 1, size=n).tolist()
    lens[n // 3] = long_len
    return lens


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_many_segments_packed_grid(causal):
    # 200 segments (lengths 0..100, one of 1000, some empty): the packed grid, whose
    # per-warp prefix sum over cu_seqlens then takes seven 32-segment steps
    lens = _many_lengths(200, 100, 1000, 41)
    run_varlen(lens, lens, 2, 64, causal, seed=41)


def test_varlen_over_1024_segments_per_segment_grid():
    # more segments than the packed grid's prefix sum takes: the per-segment grid, ragged
    lens = _many_lengths(1100, 40, 300, 42)
    run_varlen(lens, lens, 2, 64, True, seed=42)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_unequal_q_k(causal):
    # Lq != Lk per sequence: bottom-right causal alignment, including fully masked rows
    # (Lq > Lk) and sequences with no keys at all.
    lens_q = [10, 290, 5, 130, 1]
    lens_k = [50, 50, 0, 400, 7]
    run_varlen(lens_q, lens_k, 2, 128, causal, seed=12)


def test_varlen_segment_isolation():
    lens = [100, 200, 150]

    def bump(k, v, cu):
        k = k.clone(); v = v.clone()
        k[cu[0]:cu[1]] = (k[cu[0]:cu[1]].float() * 3 + 1).to(k.dtype)
        v[cu[2]:cu[3]] = (v[cu[2]:cu[3]].float() - 2).to(v.dtype)
        return k, v

    o1, l1, cu = run_varlen(lens, lens, 2, 64, True, seed=13)
    o2, l2, _ = run_varlen(lens, lens, 2, 64, True, seed=13, perturb=bump)
    # The middle segment's keys/values are untouched; its outputs must be bit-identical.
    a, b = cu[1], cu[2]
    assert torch.equal(o1[a:b], o2[a:b]) and torch.equal(l1[:, a:b], l2[:, a:b])


def test_varlen64_sampled():
    w = wl.get("varlen64")
    t = wl.generate(w, with_grad_out=False)
    cu = t["cu_seqlens"].numpy()
    q, k, v = (t[x].to(DEV) for x in ("q", "k", "v"))
    cud = t["cu_seqlens"].to(DEV)
    L = max(w.seqlens)
    o, lse = fa.varlen_fwd(q, k, v, cud, cud, L, L, w.softmax_scale, True)
    assert fa.device_status() == 0
    og, lg = f64(o), f64(lse)
    qf, kf, vf = (wl.to_f64(t[x]) for x in ("q", "k", "v"))
    rng = np.random.default_rng(33)
    for s in rng.choice(64, size=6, replace=False):
        a, b = int(cu[s]), int(cu[s + 1])
        rows = wl.sample_rows(b - a, 16, 2000 + int(s))
        for h in rng.choice(w.H, size=2, replace=False):
            o_ref, lse_ref = oracle.attention_forward(qf[a:b, h], kf[a:b, h], vf[a:b, h],
                                                      w.softmax_scale, True, rows=rows)
            check_o(og[a + rows, h], o_ref, w.dtype)
            check_lse(lg[h, a + rows], lse_ref)


def test_timeout_selftest():
    # A one-CTA kernel waits on a barrier nothing arrives at, with a 2 ms bound; the
    # library must report FA_ERR_TIMEOUT and leave the context usable.
    from exact_tiled_attention_33_b200 import _lib
    lib = _lib.load()
    st = lib.fa_selftest_wait_timeout(2000, torch.cuda.current_stream().cuda_stream)
    assert st == _lib.FA_ERR_TIMEOUT
    assert fa.device_status() == 0  # cleared
    x = torch.ones(4, device=DEV)
    assert float((x * 2).sum()) == 8.0


def test_fma_pipe_exp2_accuracy():
    # The forward computes a quarter of its exponentials with its own FMA-pipe 2^x
    # (fa_selftest_exp2 evaluates it).  Check against exact 2^x (bound 1e-4 relative, the
    # fitted polynomial's 7.5e-5 plus fp32 evaluation) and against CUDA's exp2 on the GPU.
    from exact_tiled_attention_33_b200 import _lib
    lib = _lib.load()
    x = torch.linspace(-126.0, 8.0, 2_000_001, dtype=torch.float32, device=DEV)
    x = torch.cat([x, torch.tensor([-1000.0, -200.0, -126.5, 0.0, -0.5, 0.5, 7.999],
                                   device=DEV)])
    y = torch.empty_like(x)
    assert lib.fa_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(),
                                torch.cuda.current_stream().cuda_stream) == 0
    xs, ys = x.double().cpu().numpy(), y.double().cpu().numpy()
    ok = xs >= -125.0                              # results in the normal fp32 range
    rel = np.abs(ys[ok] / np.exp2(xs[ok]) - 1.0)
    assert rel.max() <= 1e-4, rel.max()
    assert np.all(np.abs(ys[~ok]) <= 2.0 ** -124)  # clamped / denormal boundary: ~1e-38
    cuda = torch.exp2(x).double().cpu().numpy()
    assert np.abs(ys[ok] / cuda[ok] - 1.0).max() <= 1.2e-4


def test_call_from_fresh_host_thread():
    # A host thread that has made no CUDA runtime call (as autograd worker threads may
    # not have) can call the library: it makes the device context current itself.
    import threading
    w = wl.custom("thread", B=1, N=200, H=2, d=64, causal=True, seed=14)
    t = wl.generate(w, with_grad_out=False)
    q, k, v = (t[x].to(DEV) for x in ("q", "k", "v"))
    o_ref, l_ref = fa.fwd(q, k, v, None, True)
    o, lse = torch.empty_like(o_ref), torch.empty_like(l_ref)
    torch.cuda.synchronize()
    err = []

    def worker():
        try:
            fa.fwd(q, k, v, None, True, out=o, lse=lse)
        except Exception as e:  # reported to the main thread
            err.append(e)

    th = threading.Thread(target=worker)
    th.start()
    th.join()
    assert not err, err
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_malformed_cu_seqlens_are_reported_not_followed():
    # cu_seqlens live on the device, so the host cannot check them: a segment beyond the
    # packed total, or longer than max_seqlen, is skipped by the kernels and reported as
    # FA_ERR_INVALID_ARG; nothing is read or written out of bounds.
    from exact_tiled_attention_33_b200 import _lib
    H, d = 2, 64
    q = torch.randn((300, H, d), device=DEV).to(torch.bfloat16)
    k, v = torch.randn_like(q), torch.randn_like(q)
    o, obuf = guarded_empty(q.shape, q.dtype, DEV)
    lse, lbuf = guarded_empty((H, 300), torch.float32, DEV)
    bad_total = torch.tensor([0, 100, 400], dtype=torch.int32, device=DEV)   # 400 > 300 rows
    fa.varlen_fwd(q, k, v, bad_total, bad_total, 300, 300, None, True, out=o, lse=lse)
    assert fa.device_status() == _lib.FA_ERR_INVALID_ARG
    assert guard_intact(obuf, o.numel()) and guard_intact(lbuf, lse.numel())
    short = torch.tensor([0, 100, 300], dtype=torch.int32, device=DEV)       # 200 > max 128
    fa.varlen_fwd(q, k, v, short, short, 128, 128, None, True, out=o, lse=lse)
    assert fa.device_status() == _lib.FA_ERR_INVALID_ARG
    o2, lse2 = fa.varlen_fwd(q, k, v, short, short, 200, 200, None, True)
    do = torch.randn_like(q)
    fa.varlen_bwd(q, k, v, o2, lse2, do, bad_total, bad_total, 300, 300, None, True)
    assert fa.device_status() == _lib.FA_ERR_INVALID_ARG
    fa.varlen_bwd(q, k, v, o2, lse2, do, short, short, 200, 200, None, True)
    assert fa.device_status() == 0  # well-formed again
