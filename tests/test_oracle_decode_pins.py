"""Pins of the oracle's KV-cache decode step (contiguous and paged caches) against facts
outside the oracle: a hand-worked cache, reduction to the already pinned dense causal
attention when the cache holds exactly the query tokens, invariance of a paged cache
under any placement of its pages, the pages' split-and-merge rule for partial softmax
statistics (the step a split-KV decode uses), and that cache rows past a sequence's
length are never read."""

import math

import numpy as np
import pytest

import oracle

LN3 = math.log(3.0)


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_worked_decode():
    # One sequence, one head, d = 1, scale 1: cache keys [0, ln3, 5], values [4, 8, 100],
    # cache length 2 (the third row is not part of the sequence), one new query q = 1
    # at position 1: weights [1/4, 3/4], O = 7, LSE = ln4, causal or not.
    q = np.ones((1, 1, 1, 1))
    k = np.array([0.0, LN3, 5.0]).reshape(1, 3, 1, 1)
    v = np.array([4.0, 8.0, 100.0]).reshape(1, 3, 1, 1)
    for causal in (False, True):
        o, lse = oracle.decode_attention(q, k, v, [2], 1.0, causal)
        assert o[0, 0, 0, 0] == pytest.approx(7.0, abs=1e-14)
        assert lse[0, 0, 0] == pytest.approx(math.log(4.0), abs=1e-14)


def test_decode_of_whole_sequence_is_dense_causal():
    # With the cache holding exactly the Nq query tokens' keys, a decode step is dense
    # causal attention over those tokens.
    B, N, H, d = 2, 9, 3, 4
    q = rnd((B, N, H, d), 1); k = rnd((B, N, H, d), 2); v = rnd((B, N, H, d), 3)
    o, lse = oracle.decode_attention(q, k, v, [N, N], 0.5, True)
    o2, l2 = oracle.attention_forward_bhsd(q, k, v, 0.5, True)
    np.testing.assert_allclose(o, o2, atol=1e-15)
    np.testing.assert_allclose(lse, l2, atol=1e-15)


@pytest.mark.parametrize("page_size", [1, 2, 4, 16])
def test_paged_cache_placement_invariance(page_size):
    B, cap, H, d, Nq = 3, 32, 2, 4, 2
    lens = [32, 7, 19]
    q = rnd((B, Nq, H, d), 4); k = rnd((B, cap, H, d), 5); v = rnd((B, cap, H, d), 6)
    o_ref, l_ref = oracle.decode_attention(q, k, v, lens, 0.7, True)
    blocks = cap // page_size
    num_pages = B * blocks + 5
    perm = np.random.default_rng(7).permutation(num_pages)[:B * blocks].reshape(B, blocks)
    kp = np.full((num_pages, page_size, H, d), np.nan)  # unused pages hold NaN
    vp = np.full((num_pages, page_size, H, d), np.nan)
    for b in range(B):
        for i in range(blocks):
            rows = slice(i * page_size, (i + 1) * page_size)
            kp[perm[b, i]] = k[b, rows]
            vp[perm[b, i]] = v[b, rows]
    o, lse = oracle.decode_attention(q, kp, vp, lens, 0.7, True, block_table=perm)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(lse, l_ref)


def test_rows_past_the_length_are_not_read():
    B, cap, H, d = 2, 20, 2, 4
    q = rnd((B, 1, H, d), 8); k = rnd((B, cap, H, d), 9); v = rnd((B, cap, H, d), 10)
    lens = [11, 3]
    o, lse = oracle.decode_attention(q, k, v, lens, 0.4, False)
    k2, v2 = k.copy(), v.copy()
    for b, L in enumerate(lens):
        k2[b, L:] = np.nan
        v2[b, L:] = np.inf
    o2, l2 = oracle.decode_attention(q, k2, v2, lens, 0.4, False)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, l2)


@pytest.mark.parametrize("split", [1, 5, 13])
def test_split_cache_merges_by_the_pages_rule(split):
    # Attention over a cache split in two parts, merged with the running-max / rescaled-sum
    # rule of the page "FlashAttention实战：如何在A100上实现3倍加速的Transformer训练" §3.1
    # (m = max(m1, m2); l = e^(m1-m) l1 + e^(m2-m) l2; O = (e^(m1-m) l1 O1 + e^(m2-m) l2 O2)/l),
    # equals attention over the whole cache.  In LSE form: weights e^(LSE_s - LSE).
    L, H, d = 20, 2, 4
    q = rnd((1, 1, H, d), 11); k = rnd((1, L, H, d), 12); v = rnd((1, L, H, d), 13)
    o, lse = oracle.decode_attention(q, k, v, [L], 0.8, False)
    for h in range(H):
        o1, l1 = oracle.attention_forward(q[0, :, h], k[0, :split, h], v[0, :split, h], 0.8, False)
        o2, l2 = oracle.attention_forward(q[0, :, h], k[0, split:, h], v[0, split:, h], 0.8, False)
        m = max(l1[0], l2[0])
        tot = math.exp(l1[0] - m) + math.exp(l2[0] - m)
        merged_lse = m + math.log(tot)
        merged_o = (math.exp(l1[0] - merged_lse) * o1[0] + math.exp(l2[0] - merged_lse) * o2[0])
        assert lse[0, h, 0] == pytest.approx(merged_lse, abs=1e-13)
        np.testing.assert_allclose(o[0, 0, h], merged_o, atol=1e-13)


def test_short_cache_rows_are_dead():
    # Nq > L with causal: the first Nq - L query rows sit at negative positions and see
    # no key (O = 0, LSE = +inf); the rest see a causal prefix.
    q = rnd((1, 4, 1, 3), 14); k = rnd((1, 6, 1, 3), 15); v = rnd((1, 6, 1, 3), 16)
    o, lse = oracle.decode_attention(q, k, v, [2], 1.0, True)
    assert np.all(o[0, :2] == 0) and np.all(np.isposinf(lse[0, 0, :2]))
    np.testing.assert_allclose(o[0, 2, 0], v[0, 0, 0], atol=1e-15)
    assert np.all(np.isfinite(lse[0, 0, 2:]))


def test_planted_decode_mistakes_are_caught(monkeypatch):
    """Mutants (page index and row swapped in the gather, top-left query positions) must
    fail the pins above."""
    import oracle.attn_ref as ref
    real_gather, real_fwd = ref.kv_cache_gather, ref.attention_forward

    def bad_gather(pages, row, length):
        pages = np.asarray(pages)
        idx = np.arange(length)
        ps = pages.shape[1]
        return pages[np.asarray(row)[idx % max(1, len(row))], idx // len(row) % ps]

    monkeypatch.setattr(ref, "kv_cache_gather", bad_gather)
    with pytest.raises(AssertionError):
        test_paged_cache_placement_invariance(4)
    monkeypatch.setattr(ref, "kv_cache_gather", real_gather)

    def top_left(q, k, v, scale, causal, rows=None, window=None):
        # drops the bottom-right shift: pads nothing, truncates keys to Lq
        return real_fwd(q, k[:len(q)], v[:len(q)], scale, causal, rows, window)

    monkeypatch.setattr(ref, "attention_forward", top_left)
    with pytest.raises(AssertionError):
        test_worked_decode()
    monkeypatch.setattr(ref, "attention_forward", real_fwd)
