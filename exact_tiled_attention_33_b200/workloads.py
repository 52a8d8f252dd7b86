"""Seeded synthetic workloads for exact attention.

This module only draws random inputs and describes problem sizes.  It contains no
attention arithmetic, and both the CUDA path's tests/bench and the CPU oracle's tests
take their inputs from here, so the two sides always see identical 16-bit values.

Recipe (identical for every workload):
  * a CPU ``torch.Generator`` seeded with the workload's seed;
  * ``torch.randn`` in float32 drawn in the order Q, K, V, dO (standard normal, the
    i.i.d. N(0, 1) inputs the workloads call for);
  * optional multiplication of Q and K by ``qk_mult`` (the "peaky softmax" stress case);
  * a cast to the workload dtype (bf16 or fp16) on the CPU.
The exact 16-bit tensors are what the GPU receives; their float64 upcast is what the
oracle receives.

Varlen lengths for the 64-sequence case are drawn with
``numpy.random.default_rng(3).integers(64, 4097, size=64)`` (uniform on [64, 4096]).

Problem sizes follow the shapes the pages use: the A100 table of the page
"FlashAttention实战：如何在A100上实现3倍加速的Transformer训练" §6 (B=8, H=16, d=64,
N=1K..4K), the Llama-style head and 16K benchmark of "FlashAttention-2的核心设计原理"
(B=4/2, H=32, d=128) and its varlen example (lengths 128/256/512, cu_seqlens
[0, 128, 384, 896]).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    d: int
    dtype: str                       # "bf16" | "fp16"
    causal: bool
    seed: int
    B: int = 0                       # dense only
    N: int = 0                       # dense only
    seqlens: Optional[tuple] = None  # varlen only
    qk_mult: float = 1.0
    scale: Optional[float] = None    # default 1/sqrt(d)
    window: Optional[tuple] = None   # sliding window (left, right); None: `causal` decides
    fp8: bool = False                # q, k, v quantised to E4M3 (dtype: the output's format)

    @property
    def varlen(self) -> bool:
        return self.seqlens is not None

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16

    @property
    def total(self) -> int:
        return int(sum(self.seqlens)) if self.varlen else self.B * self.N

    def cu_seqlens(self) -> np.ndarray:
        assert self.varlen
        return np.concatenate([[0], np.cumsum(self.seqlens)]).astype(np.int32)

    def fwd_flops(self) -> float:
        """4·B·H·N²·d forward FLOPs, halved when causal; varlen sums per sequence.  With a
        sliding window: 4·d FLOPs per allowed (query, key) pair, counted exactly."""
        lens = self.seqlens if self.varlen else (self.N,) * self.B
        if self.window is not None:
            return sum(4.0 * self.H * self.d * window_pairs(L, L, self.window) for L in lens)
        f = sum(4.0 * self.H * L * L * self.d for L in lens)
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        return 2.5 * self.fwd_flops()

    def shape(self):
        if self.varlen:
            return (self.total, self.H, self.d)
        return (self.B, self.N, self.H, self.d)

    def describe(self) -> dict:
        out = {"workload": self.name, "H": self.H, "d": self.d, "dtype": self.dtype,
               "causal": self.causal, "seed": self.seed, "scale": self.softmax_scale}
        if self.varlen:
            out.update(num_seqs=len(self.seqlens), total_tokens=self.total,
                       max_seqlen=int(max(self.seqlens)))
        else:
            out.update(B=self.B, N=self.N)
        if self.qk_mult != 1.0:
            out["qk_mult"] = self.qk_mult
        if self.window is not None:
            out["window"] = list(self.window)
        if self.fp8:
            out["inputs"] = "e4m3, per-tensor descale"
        return out


def window_pairs(Lq: int, Lk: int, window) -> int:
    """Number of (query, key) pairs a sliding window (left, right) admits in one sequence
    (bottom-right aligned; a negative bound is no bound).  Used to size FLOP counts."""
    left, right = window
    diag = Lk - Lq
    total = 0
    for i in range(Lq):
        lo = 0 if left < 0 else max(0, i + diag - left)
        hi = Lk - 1 if right < 0 else min(Lk - 1, i + diag + right)
        total += max(0, hi - lo + 1)
    return total


def varlen_lengths_64(seed: int = 3) -> tuple:
    rng = np.random.default_rng(seed)
    return tuple(int(x) for x in rng.integers(64, 4097, size=64))


def _registry():
    w = {}

    def add(x: Workload):
        w[x.name] = x

    for causal in (False, True):
        c = "causal" if causal else "noncausal"
        add(Workload(f"tiny_{c}", B=1, H=2, N=128, d=64, dtype="bf16", causal=causal, seed=0,
                     scale=1.0 / 8.0))
    for N in (1024, 2048, 4096):
        add(Workload(f"a100table_N{N}", B=8, H=16, N=N, d=64, dtype="bf16", causal=True,
                     seed=1, scale=1.0 / 8.0))
    for causal in (False, True):
        c = "causal" if causal else "noncausal"
        add(Workload(f"llama_{c}", B=4, H=32, N=4096, d=128, dtype="fp16", causal=causal,
                     seed=2))
    add(Workload("varlen3", H=32, d=128, dtype="bf16", causal=True, seed=3,
                 seqlens=(128, 256, 512)))
    add(Workload("varlen64", H=32, d=128, dtype="bf16", causal=True, seed=3,
                 seqlens=varlen_lengths_64(3)))
    for causal in (False, True):
        c = "causal" if causal else "noncausal"
        add(Workload(f"long_{c}", B=2, H=32, N=16384, d=128, dtype="bf16", causal=causal,
                     seed=4))
        add(Workload(f"long_peaky_{c}", B=2, H=32, N=16384, d=128, dtype="bf16",
                     causal=causal, seed=4, qk_mult=4.0))
    # FP8 (E4M3) inputs at the long-context size, per-tensor scales
    for causal in (False, True):
        c = "causal" if causal else "noncausal"
        add(Workload(f"fp8_long_{c}", B=2, H=32, N=16384, d=128, dtype="bf16", causal=causal,
                     seed=4, fp8=True))
    # sliding-window (local) attention at the long-context size: each query sees the 4096
    # keys ending at its own position (a causal window of 4096), and a symmetric window
    add(Workload("long_local_w4096", B=2, H=32, N=16384, d=128, dtype="bf16", causal=True,
                 seed=4, window=(4095, 0)))
    add(Workload("long_local_sym512", B=2, H=32, N=16384, d=128, dtype="bf16", causal=False,
                 seed=4, window=(256, 256)))
    # profiling size of the long-context kernel path: inputs larger than L2 (4 x 67 MB),
    # about 1 GB on the device in total
    add(Workload("profile_causal_8k", B=1, H=32, N=8192, d=128, dtype="bf16", causal=True,
                 seed=4))
    return w


WORKLOADS = _registry()


def get(name: str) -> Workload:
    return WORKLOADS[name]


def custom(name="custom", *, B=1, N=128, H=1, d=64, dtype="bf16", causal=False, seed=0,
           seqlens=None, qk_mult=1.0, scale=None, window=None, fp8=False) -> Workload:
    """An ad-hoc workload (ragged sizes, edge cases) built with the same recipe."""
    window = None if window is None else (int(window[0]), int(window[1]))
    if seqlens is not None:
        return Workload(name, H=H, d=d, dtype=dtype, causal=causal, seed=seed,
                        seqlens=tuple(int(x) for x in seqlens), qk_mult=qk_mult, scale=scale,
                        window=window, fp8=fp8)
    return Workload(name, B=B, N=N, H=H, d=d, dtype=dtype, causal=causal, seed=seed,
                    qk_mult=qk_mult, scale=scale, window=window, fp8=fp8)


def generate(w: Workload, with_grad_out: bool = True):
    """Return dict of CPU 16-bit tensors q, k, v (and do) with the workload's shape."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    shape = w.shape()
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    out = {}
    if w.qk_mult != 1.0:
        q = q * w.qk_mult
        k = k * w.qk_mult
    out["q"] = q.to(w.torch_dtype)
    out["k"] = k.to(w.torch_dtype)
    out["v"] = v.to(w.torch_dtype)
    if with_grad_out:
        out["do"] = torch.randn(shape, generator=g, dtype=torch.float32).to(w.torch_dtype)
    if w.varlen:
        out["cu_seqlens"] = torch.from_numpy(w.cu_seqlens())
    if w.fp8:
        # per-tensor scaling to the E4M3 range: descale = amax / 448, codes = x / descale
        # rounded to nearest (PyTorch's float8_e4m3fn cast).  The 16-bit q, k, v above are
        # replaced by the dequantised values rounded to 16 bits, a view for callers that
        # want one; the FP8 kernels take the codes and descales, and the parity tests give
        # the oracle the codes and descales too (exact in fp64)
        for name, x in (("q", q), ("k", k), ("v", v)):
            descale = float(x.abs().max()) / 448.0
            x8 = (x / descale).to(torch.float8_e4m3fn)
            out[name + "8"] = x8
            out[name + "_descale"] = descale
            out[name] = (x8.to(torch.float32) * descale).to(w.torch_dtype)
    return out


# ------------------------------------------------------------------ KV-cache decode
@dataclass(frozen=True)
class DecodeWorkload:
    """One decode step: Nq new query tokens per sequence against its cached K/V.

    Recipe: a CPU torch.Generator seeded with `seed`; randn fp32 in the order q, K cache,
    V cache, cast to the dtype.  Contiguous caches are [B, capacity, H, d]; paged caches
    are [num_pages, page_size, H, d] with a block table that is a seeded permutation of
    the pages (numpy default_rng(seed + 1)), two spare pages left unused.  Cache rows past
    a sequence's length, and unused pages, hold NaN: a correct kernel never reads them.
    """
    name: str
    B: int
    Nq: int
    H: int
    d: int
    dtype: str
    causal: bool
    seed: int
    cache_lens: tuple
    capacity: int
    page_size: int = 0               # 0: contiguous cache
    scale: Optional[float] = None

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16

    @property
    def max_blocks(self) -> int:
        return -(-self.capacity // self.page_size) if self.page_size else 0

    def window(self):
        return (-1, 0) if self.causal else (-1, -1)

    def flops(self) -> float:
        """4·d FLOPs per allowed (query, key) pair, summed over sequences and heads."""
        w = self.window()
        return sum(4.0 * self.H * self.d * window_pairs(self.Nq, L, w) for L in self.cache_lens)

    def bytes_moved(self) -> float:
        """Algorithmic HBM bytes of one step: the cached K and V rows of every sequence
        (read once), q read, O written, LSE written."""
        el = 2
        kv = 2 * sum(self.cache_lens) * self.H * self.d * el
        qo = 2 * self.B * self.Nq * self.H * self.d * el
        return float(kv + qo + 4 * self.B * self.H * self.Nq)

    def describe(self) -> dict:
        out = {"workload": self.name, "B": self.B, "Nq": self.Nq, "H": self.H, "d": self.d,
               "dtype": self.dtype, "causal": self.causal, "seed": self.seed,
               "scale": self.softmax_scale, "capacity": self.capacity,
               "cache_tokens": int(sum(self.cache_lens)),
               "max_cache_len": int(max(self.cache_lens))}
        out["layout"] = f"paged (page_size {self.page_size})" if self.page_size else "contiguous"
        return out


def generate_decode(w: DecodeWorkload) -> dict:
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    q = torch.randn((w.B, w.Nq, w.H, w.d), generator=g, dtype=torch.float32).to(w.torch_dtype)
    lens = torch.tensor(w.cache_lens, dtype=torch.int32)
    k = torch.randn((w.B, w.capacity, w.H, w.d), generator=g, dtype=torch.float32)
    v = torch.randn((w.B, w.capacity, w.H, w.d), generator=g, dtype=torch.float32)
    for b, L in enumerate(w.cache_lens):
        k[b, L:] = float("nan")
        v[b, L:] = float("nan")
    k, v = k.to(w.torch_dtype), v.to(w.torch_dtype)
    out = {"q": q, "cache_seqlens": lens}
    if not w.page_size:
        out["k_cache"], out["v_cache"] = k, v
        return out
    ps, mb = w.page_size, w.max_blocks
    num_pages = w.B * mb + 2
    perm = np.random.default_rng(w.seed + 1).permutation(num_pages)[:w.B * mb].reshape(w.B, mb)
    pad = mb * ps - w.capacity
    kp = torch.full((num_pages, ps, w.H, w.d), float("nan"), dtype=w.torch_dtype)
    vp = torch.full((num_pages, ps, w.H, w.d), float("nan"), dtype=w.torch_dtype)
    kk = torch.nn.functional.pad(k, (0, 0, 0, 0, 0, pad), value=float("nan")) if pad else k
    vv = torch.nn.functional.pad(v, (0, 0, 0, 0, 0, pad), value=float("nan")) if pad else v
    idx = torch.from_numpy(perm.reshape(-1).astype(np.int64))
    kp[idx] = kk.reshape(w.B * mb, ps, w.H, w.d)
    vp[idx] = vv.reshape(w.B * mb, ps, w.H, w.d)
    out["k_pages"], out["v_pages"] = kp, vp
    out["block_table"] = torch.from_numpy(perm.astype(np.int32))
    return out


def _decode_registry():
    w = {}
    lens16 = tuple(int(x) for x in np.random.default_rng(5).integers(1, 16385, size=16))
    for x in (
        # long-context single-token decode, contiguous cache (B=8, H=32, d=128, 16K cached)
        DecodeWorkload("decode_b8_l16k", B=8, Nq=1, H=32, d=128, dtype="bf16", causal=True,
                       seed=6, cache_lens=(16384,) * 8, capacity=16384),
        # paged cache, ragged lengths uniform on [1, 16384], pages of 256 tokens
        DecodeWorkload("decode_paged_ragged", B=16, Nq=1, H=32, d=128, dtype="bf16",
                       causal=True, seed=7, cache_lens=lens16, capacity=16384, page_size=256),
        # four new tokens per step (causal among themselves), 8K cached
        DecodeWorkload("decode_q4_l8k", B=8, Nq=4, H=32, d=128, dtype="bf16", causal=True,
                       seed=8, cache_lens=(8192,) * 8, capacity=8192),
    ):
        w[x.name] = x
    return w


DECODE_WORKLOADS = _decode_registry()


def get_decode(name: str) -> DecodeWorkload:
    return DECODE_WORKLOADS[name]


def sample_rows(n_rows: int, k: int, seed: int) -> np.ndarray:
    """Sorted seeded subset of query/key rows, always containing the tile and causal
    boundaries 0, 1, 127, 128 and n_rows-1 (when they exist)."""
    rng = np.random.default_rng(seed)
    base = {0, 1, 127, 128, n_rows - 1}
    base = {r for r in base if 0 <= r < n_rows}
    k = min(k, n_rows)
    pick = set(int(x) for x in rng.choice(n_rows, size=k, replace=False))
    return np.array(sorted(pick | base), dtype=np.int64)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()
