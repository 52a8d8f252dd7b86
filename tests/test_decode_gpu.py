"""GPU parity of the KV-cache decode step — fa_decode (contiguous cache) and
fa_decode_paged (block table) through the C ABI — against the oracle's decode_attention
on seeded inputs, with the forward tolerances (O 1e-2, LSE 1e-3).  Cases cover Nq from 1
to 16, empty and one-row caches, lengths on and around the 128-key tile, many splits
merged by the combine kernel and a single split written directly, page sizes 16..256,
causal and non-causal, fp16 and bf16, d = 64 and 128.  Cache rows past each length and
unused pages hold NaN, so any read of them shows up in the output."""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_33_b200 import _lib
from exact_tiled_attention_33_b200 import attention as fa
from exact_tiled_attention_33_b200 import workloads as wl
from tests.parity import check_lse, check_o, f64, guard_intact, guarded_empty

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run(w, heads=None):
    g = wl.generate_decode(w)
    q = g["q"].to(DEV)
    lens = g["cache_seqlens"].to(DEV)
    B, Nq, H, d = q.shape
    o, ob = guarded_empty(q.shape, q.dtype, DEV)
    lse, lb = guarded_empty((B, H, Nq), torch.float32, DEV)
    max_len = max(w.cache_lens) if w.cache_lens else 0
    if w.page_size:
        kp, vp, bt = g["k_pages"].to(DEV), g["v_pages"].to(DEV), g["block_table"].to(DEV)
        fa.decode_paged(q, kp, vp, bt, lens, max_len, w.softmax_scale, w.causal, out=o, lse=lse)
    else:
        kc, vc = g["k_cache"].to(DEV), g["v_cache"].to(DEV)
        fa.decode(q, kc, vc, lens, max_len, w.softmax_scale, w.causal, out=o, lse=lse)
    assert fa.device_status() == 0
    assert guard_intact(ob, o.numel()) and guard_intact(lb, lse.numel())
    og, lg = f64(o), f64(lse)
    qf = wl.to_f64(g["q"])
    for b in range(B):
        L = w.cache_lens[b]
        if w.page_size:
            # the oracle's gather is plain indexing: run it on the raw 16-bit patterns
            row = g["block_table"][b].numpy()
            kb = torch.from_numpy(oracle.kv_cache_gather(
                g["k_pages"].view(torch.int16).numpy(), row, L)).view(q.dtype)
            vb = torch.from_numpy(oracle.kv_cache_gather(
                g["v_pages"].view(torch.int16).numpy(), row, L)).view(q.dtype)
        else:
            kb, vb = g["k_cache"][b, :L], g["v_cache"][b, :L]
        kb, vb = kb.double().numpy(), vb.double().numpy()
        for h in (range(H) if heads is None else heads):
            o_ref, l_ref = oracle.attention_forward(qf[b, :, h], kb[:, h], vb[:, h],
                                                    w.softmax_scale, w.causal)
            check_o(og[b, :, h], o_ref, w.dtype, f"O[b={b},h={h}] L={L}")
            check_lse(lg[b, h], l_ref, f"LSE[b={b},h={h}] L={L}")
    return o, lse


def small(name="dec", *, B=3, Nq=1, H=2, d=128, dtype="bf16", causal=True, seed=1,
          lens=(0, 1, 300), capacity=None, page_size=0, scale=None):
    cap = capacity if capacity is not None else max(max(lens), 1)
    return wl.DecodeWorkload(name, B=B, Nq=Nq, H=H, d=d, dtype=dtype, causal=causal, seed=seed,
                             cache_lens=tuple(lens), capacity=cap, page_size=page_size,
                             scale=scale)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Nq", [1, 2, 4, 7, 16])
@pytest.mark.parametrize("causal", [True, False])
def test_contiguous(Nq, d, causal):
    lens = (0, 1, 127, 128, 129, 1000, 5)
    w = small(B=len(lens), Nq=Nq, d=d, causal=causal, seed=10 + Nq, lens=lens, capacity=1100)
    run(w)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("scale", [0.0, -0.2, 0.3])
def test_scales_and_dtypes(dtype, scale):
    w = small(B=2, Nq=3, d=64, dtype=dtype, lens=(700, 33), seed=12, scale=scale)
    run(w)


@pytest.mark.parametrize("page_size", [16, 64, 128, 256])
@pytest.mark.parametrize("Nq", [1, 5])
def test_paged(page_size, Nq):
    lens = (1, 300, 0, 129, 1024, 77)
    w = small(B=len(lens), Nq=Nq, d=128, causal=True, seed=20 + page_size, lens=lens,
              capacity=1024, page_size=page_size)
    run(w)


def test_paged_d64_fp16_noncausal():
    w = small(B=4, Nq=2, d=64, dtype="fp16", causal=False, seed=21, lens=(50, 600, 255, 256),
              capacity=640, page_size=32)
    run(w)


def test_many_splits_and_single_split():
    # B*H = 1: a 5000-key cache is cut into one split per 128-key tile and merged by the
    # combine kernel; B*H = 1280 leaves one split per (sequence, head), written directly.
    from exact_tiled_attention_33_b200 import _lib as L
    lib = L.load()
    assert lib.fa_decode_workspace_size(1, 1, 1, 128, 5000) > 0
    assert lib.fa_decode_workspace_size(40, 1, 32, 128, 5000) == 0
    run(small(B=1, H=1, Nq=2, lens=(5000,), seed=30))
    run(small(B=40, H=32, Nq=1, d=64, lens=tuple(range(1, 4001, 100)), seed=31), heads=[0, 31])


def test_shorter_than_nq_rows_are_dead():
    # cache_seqlens < Nq with causal: the first rows see no key (O = 0, LSE = +inf)
    run(small(B=2, Nq=6, lens=(2, 0), seed=32))


def test_deterministic():
    w = small(B=2, Nq=4, lens=(3000, 1500), seed=33)
    o1, l1 = run(w)
    o2, l2 = run(w)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_long_context_workload_sampled_heads():
    run(wl.get_decode("decode_b8_l16k"), heads=[0, 13, 31])


def test_paged_ragged_workload_sampled_heads():
    run(wl.get_decode("decode_paged_ragged"), heads=[0, 7, 31])


def test_multi_query_workload_sampled_heads():
    run(wl.get_decode("decode_q4_l8k"), heads=[2, 30])


def test_device_side_bound_violations_are_reported():
    # Lengths above max_seqlen_k and page ids outside the page pool cannot be checked on
    # the host; the kernel clamps / reads zeros (nothing out of bounds) and reports.
    w = small(B=2, Nq=1, lens=(200, 100), capacity=256, seed=34)
    g = wl.generate_decode(w)
    q, kc, vc = g["q"].to(DEV), g["k_cache"].to(DEV), g["v_cache"].to(DEV)
    lens = torch.tensor([200, 100], dtype=torch.int32, device=DEV)
    fa.decode(q, kc, vc, lens, max_seqlen_k=150)
    assert fa.device_status() == _lib.FA_ERR_INVALID_ARG
    assert fa.device_status() == 0  # cleared
    wp = small(B=2, Nq=1, lens=(200, 100), capacity=256, page_size=64, seed=35)
    g = wl.generate_decode(wp)
    bt = g["block_table"].clone()
    bt[1, 0] = 10_000
    fa.decode_paged(g["q"].to(DEV), g["k_pages"].to(DEV), g["v_pages"].to(DEV), bt.to(DEV),
                    g["cache_seqlens"].to(DEV), 256)
    assert fa.device_status() == _lib.FA_ERR_INVALID_ARG
    x = torch.ones(4, device=DEV)
    assert float((x * 2).sum()) == 8.0  # context still usable
