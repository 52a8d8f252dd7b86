"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or run this
module: only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code, constants or
helpers with the CUDA library.

What it computes is the plain definition of attention given as "standard attention"
on the page "FlashAttention-2的核心设计原理" (yunthe.com), section
"FlashAttention-2与标准注意力的计算对比": scores = Q Kᵀ / sqrt(d), a softmax over the
keys, output = weights · V.  It is generalised to

* an explicit ``scale`` (the pages pass softmax_scale = 1/sqrt(head_dim): page
  "FlashAttention实战：如何在A100上实现3倍加速的Transformer训练" (jsqmd.com/news/620004)
  section 4.1; any value, zero and negative included, is accepted here),
* causal masking (the ``causal=True`` flag used on both pages) read bottom-right aligned:
  key j is allowed for query i iff j <= i + (Lk - Lq); identical to the usual
  top-left rule whenever Lq == Lk,
* the log-sum-exp of each row in natural-log, scaled-score units,
  LSE_i = ln sum_j exp(scale * q_i . k_j), the O(N) statistic the backward pass keeps
  (page "Flash Attention V3：大模型训练加速与显存优化技术解析" (jsqmd.com/news/1204652)
  section 3.2: O(N) storage, recomputation in the backward pass),
* the analytic backward of O = softmax(scale Q Kᵀ) V (chain rule; the pages only say
  that the backward pass recomputes the forward: "FlashAttention-2的核心设计原理",
  section "FlashAttention-2反向传播与多GPU训练").

Fully masked rows (possible only when Lk < Lq under the bottom-right rule, or when
Lk == 0) give O = 0 and LSE = +inf, and contribute nothing to any gradient.

Every number is float64.  Large problems are evaluated one block of at most
``ROW_BLOCK`` query rows at a time: each block materialises its full row of scores
against every key, so this is still the definition (each row of a softmax is
independent of every other row), not an online or tiled reformulation.

Parity status: every function here is pinned — the dense, causal, varlen and backward
functions by tests/test_oracle_pins.py (closed forms, invariants, brute force, finite
differences, a hand-worked golden example; the batched [B, N, H, d] forward and backward
against torch autograd of the naive formula on that layout), the sliding window by
tests/test_oracle_window_pins.py, the decode step and paged gather by
tests/test_oracle_decode_pins.py, and the E4M3 decoding and FP8 forward by
tests/test_oracle_fp8_pins.py.
"""

from __future__ import annotations

import numpy as np

ROW_BLOCK = 1024


def allowed_mask(rows: np.ndarray, Lq: int, Lk: int, causal: bool, window=None) -> np.ndarray:
    """Boolean [len(rows), Lk]: which keys each listed query row may attend to.

    Causal reading (bottom-right): key j is allowed for query i iff j <= i + (Lk - Lq).
    Sliding window (w_left, w_right), the local attention the pages list without
    parameters (page "FlashAttention技术深度解析" (pwwt.cn/news/595117), CUDA backend feature
    table and "局部注意力机制"), read around the same bottom-right diagonal:
    key j is allowed iff i + diag - w_left <= j <= i + diag + w_right, diag = Lk - Lq, a
    negative bound meaning no bound on that side.  A window, when given, replaces
    `causal`; causal is the window (-1, 0).
    """
    rows = np.asarray(rows, dtype=np.int64)
    keys = np.arange(Lk, dtype=np.int64)
    if window is None:
        window = (-1, 0) if causal else (-1, -1)
    w_left, w_right = window
    center = rows[:, None] + (Lk - Lq)
    ok = np.ones((rows.shape[0], Lk), dtype=bool)
    if w_right >= 0:
        ok &= keys[None, :] <= center + w_right
    if w_left >= 0:
        ok &= keys[None, :] >= center - w_left
    return ok


def _scores(q_rows: np.ndarray, k: np.ndarray, scale: float, mask: np.ndarray) -> np.ndarray:
    """S = scale * Q_rows Kᵀ with disallowed entries set to -inf."""
    s = scale * (q_rows @ k.T)
    return np.where(mask, s, -np.inf)


def _row_softmax_stats(s: np.ndarray):
    """Row max m, row sum l = sum exp(S - m) and LSE = m + ln l of a score block.

    Rows with no allowed key get m = -inf, l = 0, LSE = +inf.
    """
    m = s.max(axis=1) if s.shape[1] > 0 else np.full(s.shape[0], -np.inf)
    dead = ~np.isfinite(m)
    m_safe = np.where(dead, 0.0, m)
    e = np.exp(s - m_safe[:, None])  # exp(-inf) = 0 for masked entries
    l = e.sum(axis=1)
    with np.errstate(divide="ignore"):
        lse = np.where(dead, np.inf, m_safe + np.log(np.where(dead, 1.0, l)))
    return m_safe, l, lse, e, dead


def softmax_probs(q, k, scale, causal, rows=None, window=None):
    """P = softmax(scale Q Kᵀ) for the listed query rows: [len(rows), Lk] float64.

    Fully masked rows are all zero.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    Lq, Lk = q.shape[0], k.shape[0]
    rows = np.arange(Lq) if rows is None else np.asarray(rows, dtype=np.int64)
    s = _scores(q[rows], k, scale, allowed_mask(rows, Lq, Lk, causal, window))
    _, l, _, e, dead = _row_softmax_stats(s)
    return e / np.where(dead, 1.0, l)[:, None]


def attention_forward(q, k, v, scale, causal, rows=None, window=None):
    """O and LSE of one (batch, head) or one packed segment.

    q: [Lq, d], k: [Lk, d], v: [Lk, dv] (any float dtype; upcast to float64).
    rows: optional sorted query-row indices; only those rows are evaluated.
    window: optional (w_left, w_right) sliding window (see allowed_mask).
    Returns (O [n_rows, dv], LSE [n_rows]) in float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Lq, Lk = q.shape[0], k.shape[0]
    rows = np.arange(Lq) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((rows.shape[0], v.shape[1]), dtype=np.float64)
    lse = np.zeros(rows.shape[0], dtype=np.float64)
    for b0 in range(0, rows.shape[0], ROW_BLOCK):
        r = rows[b0:b0 + ROW_BLOCK]
        s = _scores(q[r], k, scale, allowed_mask(r, Lq, Lk, causal, window))
        _, l, blk_lse, e, dead = _row_softmax_stats(s)
        p = e / np.where(dead, 1.0, l)[:, None]
        out[b0:b0 + r.shape[0]] = p @ v
        lse[b0:b0 + r.shape[0]] = blk_lse
    return out, lse


def attention_backward(q, k, v, do, scale, causal, dq_rows=None, dkv_rows=None, window=None):
    """Analytic gradients of O = softmax(scale Q Kᵀ) V for one (batch, head) / segment.

    With P the softmax weights and D_i = sum_c dO_ic O_ic (O from this oracle, float64):
      dV = Pᵀ dO,  dP = dO Vᵀ,  dS = P ∘ (dP − D),  dQ = scale dS K,  dK = scale dSᵀ Q.

    dq_rows: query rows whose dQ is wanted (default: all).
    dkv_rows: key rows whose dK, dV are wanted (default: all).
    Returns (dQ [len(dq_rows), d], dK [len(dkv_rows), d], dV [len(dkv_rows), dv]).

    Every entry of P used here is exp(S_ij − LSE_i) with LSE from the full row of
    scores, i.e. the softmax definition itself; dK/dV rows need the statistics of
    every query row, which are computed block by block.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    Lq, Lk = q.shape[0], k.shape[0]
    dq_rows = np.arange(Lq) if dq_rows is None else np.asarray(dq_rows, dtype=np.int64)
    dkv_rows = np.arange(Lk) if dkv_rows is None else np.asarray(dkv_rows, dtype=np.int64)

    # dQ rows: each needs its own full row of P and dP.
    dq = np.zeros((dq_rows.shape[0], q.shape[1]), dtype=np.float64)
    for b0 in range(0, dq_rows.shape[0], ROW_BLOCK):
        r = dq_rows[b0:b0 + ROW_BLOCK]
        p = softmax_probs(q, k, scale, causal, rows=r, window=window)
        o = p @ v
        d_row = (do[r] * o).sum(axis=1)
        dp = do[r] @ v.T
        ds = p * (dp - d_row[:, None])
        dq[b0:b0 + r.shape[0]] = scale * (ds @ k)

    # dK / dV rows: need P[:, keys] for every query row, hence every row's LSE and D.
    dk = np.zeros((dkv_rows.shape[0], k.shape[1]), dtype=np.float64)
    dv = np.zeros((dkv_rows.shape[0], v.shape[1]), dtype=np.float64)
    if dkv_rows.shape[0] > 0 and Lq > 0:
        for b0 in range(0, Lq, ROW_BLOCK):
            r = np.arange(b0, min(Lq, b0 + ROW_BLOCK))
            mask = allowed_mask(r, Lq, Lk, causal, window)
            s_full = _scores(q[r], k, scale, mask)
            _, l, lse, e, dead = _row_softmax_stats(s_full)
            p_full = e / np.where(dead, 1.0, l)[:, None]
            o = p_full @ v
            d_row = (do[r] * o).sum(axis=1)
            p = p_full[:, dkv_rows]
            dp = do[r] @ v[dkv_rows].T
            ds = p * (dp - d_row[:, None])
            dv += p.T @ do[r]
            dk += scale * (ds.T @ q[r])
    return dq, dk, dv


def attention_forward_bhsd(q, k, v, scale, causal, window=None):
    """Dense batched forward over the pages' [batch, seqlen, heads, head_dim] layout.

    Returns O [B, N, H, d] and LSE [B, H, N] (float64).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, H, _ = q.shape
    out = np.zeros(q.shape[:3] + (v.shape[3],), dtype=np.float64)
    lse = np.zeros((B, H, N), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            o, l = attention_forward(q[b, :, h], k[b, :, h], v[b, :, h], scale, causal,
                                     window=window)
            out[b, :, h] = o
            lse[b, h] = l
    return out, lse


def attention_backward_bhsd(q, k, v, do, scale, causal, window=None):
    """Dense batched backward over [batch, seqlen, heads, head_dim]: (dQ, dK, dV)."""
    q = np.asarray(q, dtype=np.float64)
    B, _, H, _ = q.shape
    dq = np.zeros(q.shape, dtype=np.float64)
    dk = np.zeros(np.shape(k), dtype=np.float64)
    dv = np.zeros(np.shape(v), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            a, bb, c = attention_backward(q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h],
                                          scale, causal, window=window)
            dq[b, :, h], dk[b, :, h], dv[b, :, h] = a, bb, c
    return dq, dk, dv


def varlen_attention_forward(q, k, v, cu_seqlens_q, cu_seqlens_k, scale, causal, window=None):
    """Packed variable-length forward: [total, H, d] tensors, one segment per sequence.

    Segment s holds query rows cu_seqlens_q[s]:cu_seqlens_q[s+1] and key/value rows
    cu_seqlens_k[s]:cu_seqlens_k[s+1] (flash_attn_varlen_func usage on the page
    "FlashAttention-2的核心设计原理", section "变长序列处理与flash_attn_varlen_func").  No key outside a query's own
    segment takes part.  Returns O [total_q, H, dv] and LSE [H, total_q].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    total_q, H, _ = q.shape
    out = np.zeros((total_q, H, v.shape[2]), dtype=np.float64)
    lse = np.zeros((H, total_q), dtype=np.float64)
    for s in range(len(cu_seqlens_q) - 1):
        q0, q1 = int(cu_seqlens_q[s]), int(cu_seqlens_q[s + 1])
        k0, k1 = int(cu_seqlens_k[s]), int(cu_seqlens_k[s + 1])
        for h in range(H):
            o, l = attention_forward(q[q0:q1, h], k[k0:k1, h], v[k0:k1, h], scale, causal,
                                     window=window)
            out[q0:q1, h] = o
            lse[h, q0:q1] = l
    return out, lse


def varlen_attention_backward(q, k, v, do, cu_seqlens_q, cu_seqlens_k, scale, causal,
                              window=None):
    """Packed variable-length backward: (dQ [total_q,H,d], dK [total_k,H,d], dV)."""
    q = np.asarray(q, dtype=np.float64)
    dq = np.zeros(q.shape, dtype=np.float64)
    dk = np.zeros(np.shape(k), dtype=np.float64)
    dv = np.zeros(np.shape(v), dtype=np.float64)
    H = q.shape[1]
    for s in range(len(cu_seqlens_q) - 1):
        q0, q1 = int(cu_seqlens_q[s]), int(cu_seqlens_q[s + 1])
        k0, k1 = int(cu_seqlens_k[s]), int(cu_seqlens_k[s + 1])
        for h in range(H):
            a, b, c = attention_backward(q[q0:q1, h], k[k0:k1, h], v[k0:k1, h],
                                         do[q0:q1, h], scale, causal, window=window)
            dq[q0:q1, h], dk[k0:k1, h], dv[k0:k1, h] = a, b, c
    return dq, dk, dv


# ------------------------------------------------------------------ KV-cache decode
# The pages list KV caches for incremental decoding and paged KV caches as supported
# features without giving their interface (page "FlashAttention技术深度解析"
# (pwwt.cn/news/595117): Hopper row of the CUDA backend feature table, the causal-mask
# section on KV-cache updates and incremental decoding, and the section on KV-cache
# management with paged caches).  Read here as: one decode step attends Nq new query
# tokens per sequence to that sequence's cached keys and values; the new tokens are the
# last Nq positions of the cache, so masks are bottom-right aligned as everywhere else.

def kv_cache_gather(pages, block_table_row, length):
    """Rows 0..length-1 of one sequence's cache, from a paged cache.

    pages: [num_pages, page_size, H, d]; block_table_row[i] is the page that holds the
    sequence's rows i*page_size .. (i+1)*page_size - 1.  Returns [length, H, d].
    """
    pages = np.asarray(pages)
    page_size = pages.shape[1]
    idx = np.arange(length, dtype=np.int64)
    table = np.asarray(block_table_row, dtype=np.int64)
    return pages[table[idx // page_size], idx % page_size]


def decode_attention(q, k_cache, v_cache, cache_seqlens, scale, causal, block_table=None,
                     window=None):
    """One decode step over a KV cache: O [B, Nq, H, d] and LSE [B, H, Nq] (float64).

    q: [B, Nq, H, d].  Contiguous cache (block_table None): k_cache, v_cache are
    [B, capacity, H, d] and sequence b holds rows 0..cache_seqlens[b]-1.  Paged cache:
    k_cache, v_cache are [num_pages, page_size, H, d] and block_table [B, max_blocks]
    maps each sequence's logical pages to physical ones.  Rows of the cache at or past
    cache_seqlens[b] are never read.  Query row r of sequence b sits at position
    cache_seqlens[b] - Nq + r; `causal` / `window` are applied as in attention_forward.
    """
    q = np.asarray(q, dtype=np.float64)
    B, Nq, H, d = q.shape
    out = np.zeros((B, Nq, H, d), dtype=np.float64)
    lse = np.zeros((B, H, Nq), dtype=np.float64)
    for b in range(B):
        L = int(cache_seqlens[b])
        if block_table is None:
            kb = np.asarray(k_cache[b, :L], dtype=np.float64)
            vb = np.asarray(v_cache[b, :L], dtype=np.float64)
        else:
            kb = np.asarray(kv_cache_gather(k_cache, block_table[b], L), dtype=np.float64)
            vb = np.asarray(kv_cache_gather(v_cache, block_table[b], L), dtype=np.float64)
        for h in range(H):
            o, l = attention_forward(q[b, :, h], kb[:, h], vb[:, h], scale, causal,
                                     window=window)
            out[b, :, h] = o
            lse[b, h] = l
    return out, lse


# ------------------------------------------------------------------ FP8 (e4m3) inputs
# The pages credit FP8 tensor-core support to Hopper and quote FP8 attention at over 1.2
# PFLOPS with an 8-bit quantization strategy (page "FlashAttention实战：如何在A100上实现3倍
# 加速的Transformer训练" §7; page "Flash Attention V3：大模型训练加速与显存优化技术解析"
# §2.1; page "FlashAttention技术深度解析", CUDA backend feature table) without fixing a
# format or scaling.  Read here as the OCP FP8 E4M3 format the tensor cores take, one
# dequantisation factor per tensor: the attention inputs are q = sq·Q8, k = sk·K8, v = sv·V8.

def e4m3_to_float(codes):
    """Decode FP8 E4M3 bytes to float64: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
    bits; exponent 0 is subnormal (m · 2^-9); no infinities; S.1111.111 is NaN.
    Largest finite magnitude 448."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def attention_forward_fp8(q8, k8, v8, q_descale, k_descale, v_descale, scale, causal,
                          rows=None, window=None):
    """Attention of dequantised FP8 inputs: attention_forward(sq·Q8, sk·K8, sv·V8)."""
    q = e4m3_to_float(q8) * float(q_descale)
    k = e4m3_to_float(k8) * float(k_descale)
    v = e4m3_to_float(v8) * float(v_descale)
    return attention_forward(q, k, v, scale, causal, rows=rows, window=window)
