"""CPU checks that the seeded synthetic inputs follow the recipe stated for them (one CPU
torch.Generator per workload, randn fp32 in the order Q, K, V, dO, the peaky Q,K x4 before
the cast, the 64-sequence length draw, the FP8 per-tensor scaling, and the decode caches'
NaN padding and page permutation), so that the GPU path and the oracle keep receiving the
inputs the measurements and parity results describe."""

import numpy as np
import torch

from exact_tiled_attention_33_b200 import workloads as wl


def _draws(seed, shape, n):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return [torch.randn(shape, generator=g, dtype=torch.float32) for _ in range(n)]


def test_dense_recipe_order_and_cast():
    w = wl.get("tiny_causal")
    t = wl.generate(w)
    q, k, v, do = _draws(w.seed, w.shape(), 4)
    for name, x in zip(("q", "k", "v", "do"), (q, k, v, do)):
        assert torch.equal(t[name], x.to(torch.bfloat16)), name
    assert wl.get("llama_causal").torch_dtype == torch.float16


def test_peaky_scales_q_and_k_before_the_cast():
    w = wl.custom("peaky", B=1, N=64, H=2, d=64, causal=True, seed=9, qk_mult=4.0)
    t = wl.generate(w)
    q, k, v, do = _draws(9, w.shape(), 4)
    assert torch.equal(t["q"], (q * 4).to(torch.bfloat16))
    assert torch.equal(t["k"], (k * 4).to(torch.bfloat16))
    assert torch.equal(t["v"], v.to(torch.bfloat16)) and torch.equal(t["do"], do.to(torch.bfloat16))


def test_varlen64_lengths_and_offsets():
    w = wl.get("varlen64")
    lens = np.random.default_rng(3).integers(64, 4097, size=64)
    assert list(w.seqlens) == [int(x) for x in lens]
    cu = w.cu_seqlens()
    assert cu.dtype == np.int32 and cu[0] == 0 and np.array_equal(np.diff(cu), lens)
    assert w.total == int(lens.sum())


def test_fp8_scaling():
    w = wl.custom("fp8", B=1, N=256, H=2, d=128, causal=True, seed=11, fp8=True)
    t = wl.generate(w, with_grad_out=False)
    q, k, v = _draws(11, w.shape(), 3)
    for name, x in zip(("q", "k", "v"), (q, k, v)):
        ds = t[name + "_descale"]
        assert ds == float(x.abs().max()) / 448.0
        codes = t[name + "8"]
        assert codes.dtype == torch.float8_e4m3fn
        assert torch.equal(codes, (x / ds).to(torch.float8_e4m3fn))
        assert float(codes.to(torch.float32).abs().max()) == 448.0  # the amax maps to 448


def test_decode_caches():
    w = wl.DecodeWorkload("d", B=3, Nq=2, H=2, d=64, dtype="bf16", causal=True, seed=4,
                          cache_lens=(5, 0, 40), capacity=48)
    g = wl.generate_decode(w)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(4)
    q = torch.randn((3, 2, 2, 64), generator=gen, dtype=torch.float32)
    k = torch.randn((3, 48, 2, 64), generator=gen, dtype=torch.float32)
    v = torch.randn((3, 48, 2, 64), generator=gen, dtype=torch.float32)
    assert torch.equal(g["q"], q.to(torch.bfloat16))
    for b, L in enumerate(w.cache_lens):
        assert torch.equal(g["k_cache"][b, :L], k[b, :L].to(torch.bfloat16))
        assert torch.equal(g["v_cache"][b, :L], v[b, :L].to(torch.bfloat16))
        assert torch.isnan(g["k_cache"][b, L:].float()).all()
        assert torch.isnan(g["v_cache"][b, L:].float()).all()
    assert g["cache_seqlens"].tolist() == [5, 0, 40]


def test_paged_cache_is_a_permutation_of_the_contiguous_one():
    w = wl.DecodeWorkload("p", B=2, Nq=1, H=1, d=64, dtype="bf16", causal=True, seed=6,
                          cache_lens=(70, 33), capacity=96, page_size=32)
    g = wl.generate_decode(w)
    wc = wl.DecodeWorkload("c", B=2, Nq=1, H=1, d=64, dtype="bf16", causal=True, seed=6,
                           cache_lens=(70, 33), capacity=96)
    c = wl.generate_decode(wc)
    bt = g["block_table"].numpy()
    num_pages = g["k_pages"].shape[0]
    assert bt.dtype == np.int32 and len(set(bt.reshape(-1).tolist())) == bt.size
    assert bt.min() >= 0 and bt.max() < num_pages
    ps = w.page_size
    for b, L in enumerate(w.cache_lens):
        rows = torch.cat([g["k_pages"][bt[b, i]] for i in range(bt.shape[1])])[:L]
        assert torch.equal(rows, c["k_cache"][b, :L])
    unused = sorted(set(range(num_pages)) - set(bt.reshape(-1).tolist()))
    assert unused and all(torch.isnan(g["k_pages"][p].float()).all() for p in unused)
    assert bt.shape == (2, (w.capacity + ps - 1) // ps)
