"""Pins of the oracle's sliding-window (local) attention against facts outside the oracle.

The pages list sliding-window attention as a supported variant without fixing its
parameters (page "FlashAttention技术深度解析" (pwwt.cn/news/595117), CUDA backend
feature table and the section on local attention).  The reading pinned here: a window
(w_left, w_right) around the bottom-right-aligned diagonal, key j allowed for query i iff
i + (Lk - Lq) - w_left <= j <= i + (Lk - Lq) + w_right, a negative bound meaning no
bound on that side.  The pins are hand-worked closed forms, the special cases that
reduce to full and causal attention, a time-reversal symmetry, per-row key slicing,
a scalar-loop writing, finite differences, and planted mistakes that must be caught.
"""

import math

import numpy as np
import pytest

import oracle

LN3, LN5 = math.log(3.0), math.log(5.0)


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- hand-worked cases
# d = 1, scale = 1, q = 1, keys [0, ln3, ln5] so exp(scores) = [1, 3, 5]; v = [4, 8, 16].
Q3 = np.ones((3, 1))
K3 = np.array([[0.0], [LN3], [LN5]])
V3 = np.array([[4.0], [8.0], [16.0]])


def test_worked_window_left1():
    # Window (1, 0): row 0 sees {0}; row 1 sees {0,1}: weights [1/4, 3/4];
    # row 2 sees {1,2}: weights [3/8, 5/8].
    # O = [4, (4 + 24)/4, (24 + 80)/8] = [4, 7, 13]; LSE = [0, ln4, ln8].
    # dO = 1: row 1 dS = [1/4(4-7), 3/4(8-7)] = [-3/4, 3/4];
    #         row 2 dS = [3/8(8-13), 5/8(16-13)] = [-15/8, 15/8].
    # dQ = [0, 3/4 ln3, 15/8 (ln5 - ln3)]; dK = [-3/4, 3/4 - 15/8, 15/8];
    # dV = [1 + 1/4, 3/4 + 3/8, 5/8].
    o, lse = oracle.attention_forward(Q3, K3, V3, 1.0, False, window=(1, 0))
    np.testing.assert_allclose(o[:, 0], [4.0, 7.0, 13.0], atol=1e-14)
    np.testing.assert_allclose(lse, [0.0, math.log(4), math.log(8)], atol=1e-14)
    dq, dk, dv = oracle.attention_backward(Q3, K3, V3, np.ones((3, 1)), 1.0, False,
                                           window=(1, 0))
    np.testing.assert_allclose(dq[:, 0], [0.0, 0.75 * LN3, 15 / 8 * (LN5 - LN3)], atol=1e-14)
    np.testing.assert_allclose(dk[:, 0], [-0.75, 0.75 - 15 / 8, 15 / 8], atol=1e-14)
    np.testing.assert_allclose(dv[:, 0], [1.25, 1.125, 0.625], atol=1e-14)


def test_worked_window_right1():
    # Window (0, 1): row 0 sees {0,1}: O = 7, LSE = ln4; row 1 sees {1,2}: O = 13,
    # LSE = ln8; row 2 sees {2}: O = 16, LSE = ln5.  The causal flag is ignored.
    for causal in (False, True):
        o, lse = oracle.attention_forward(Q3, K3, V3, 1.0, causal, window=(0, 1))
        np.testing.assert_allclose(o[:, 0], [7.0, 13.0, 16.0], atol=1e-14)
        np.testing.assert_allclose(lse, [math.log(4), math.log(8), LN5], atol=1e-14)


def test_worked_window_bottom_right_alignment():
    # Lq = 1, Lk = 3: the single query sits on key 2 (diag = 2).  Window (1, 0) sees
    # keys {1, 2}: O = 13, LSE = ln8.  Window (0, 0) sees key 2 only: O = 16.
    o, lse = oracle.attention_forward(Q3[:1], K3, V3, 1.0, False, window=(1, 0))
    assert o[0, 0] == pytest.approx(13.0, abs=1e-14) and lse[0] == pytest.approx(math.log(8))
    o, lse = oracle.attention_forward(Q3[:1], K3, V3, 1.0, False, window=(0, 0))
    assert o[0, 0] == pytest.approx(16.0, abs=1e-14) and lse[0] == pytest.approx(LN5)


# ---------------------------------------------------------------- special cases
@pytest.mark.parametrize("Lq,Lk", [(9, 9), (5, 11), (11, 5)])
def test_window_reduces_to_full_and_causal(Lq, Lk):
    q = rnd((Lq, 4), 1); k = rnd((Lk, 4), 2); v = rnd((Lk, 3), 3)
    full = oracle.attention_forward(q, k, v, 0.7, False)
    causal = oracle.attention_forward(q, k, v, 0.7, True)
    big = Lq + Lk
    for win, ref in (((-1, -1), full), ((big, big), full), ((big, -1), full),
                     ((-1, 0), causal), ((big, 0), causal)):
        o, lse = oracle.attention_forward(q, k, v, 0.7, False, window=win)
        np.testing.assert_allclose(o, ref[0], atol=1e-14, err_msg=str(win))
        np.testing.assert_allclose(lse, ref[1], atol=1e-14, err_msg=str(win))


@pytest.mark.parametrize("Lq,Lk", [(6, 6), (4, 9), (9, 4)])
def test_diagonal_window_picks_one_key(Lq, Lk):
    # Window (0, 0): row i sees key i + Lk - Lq alone (O = that value row, LSE = its
    # score) or nothing when that index is negative (O = 0, LSE = +inf).
    q = rnd((Lq, 4), 4); k = rnd((Lk, 4), 5); v = rnd((Lk, 3), 6)
    o, lse = oracle.attention_forward(q, k, v, 0.6, True, window=(0, 0))
    for i in range(Lq):
        j = i + Lk - Lq
        if j < 0:
            assert np.all(o[i] == 0.0) and np.isposinf(lse[i])
        else:
            np.testing.assert_allclose(o[i], v[j], atol=1e-14)
            assert lse[i] == pytest.approx(0.6 * float(q[i] @ k[j]), abs=1e-13)


@pytest.mark.parametrize("win", [(2, 0), (0, 3), (1, 4), (3, -1), (-1, 2)])
def test_time_reversal(win):
    # For Lq = Lk, reversing the order of queries and keys swaps the two sides of the
    # window: window (a, b) on (q, k, v) equals window (b, a) on the reversed sequences.
    L = 10
    q = rnd((L, 4), 7); k = rnd((L, 4), 8); v = rnd((L, 3), 9)
    o, lse = oracle.attention_forward(q, k, v, 0.9, False, window=win)
    o2, lse2 = oracle.attention_forward(q[::-1], k[::-1], v[::-1], 0.9, False,
                                        window=(win[1], win[0]))
    np.testing.assert_allclose(o, o2[::-1], atol=1e-13)
    np.testing.assert_allclose(lse, lse2[::-1], atol=1e-13)


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("Lq,Lk", [(8, 8), (5, 12), (12, 5)])
@pytest.mark.parametrize("win", [(2, 1), (0, 3), (4, 0), (3, -1), (-1, 1)])
def test_window_equals_sliced_full_attention(Lq, Lk, win):
    # Each row's windowed attention equals plain (unmasked) attention over that row's
    # contiguous slice of keys.
    q = rnd((Lq, 4), 10); k = rnd((Lk, 4), 11); v = rnd((Lk, 3), 12)
    o, lse = oracle.attention_forward(q, k, v, 0.8, False, window=win)
    for i in range(Lq):
        c = i + Lk - Lq
        lo = 0 if win[0] < 0 else max(0, c - win[0])
        hi = Lk if win[1] < 0 else min(Lk, c + win[1] + 1)
        if hi <= lo:
            assert np.all(o[i] == 0.0) and np.isposinf(lse[i])
            continue
        o1, l1 = oracle.attention_forward(q[i:i + 1], k[lo:hi], v[lo:hi], 0.8, False)
        np.testing.assert_allclose(o[i], o1[0], atol=1e-14)
        assert lse[i] == pytest.approx(l1[0], abs=1e-14)


def _loops_window(q, k, v, scale, win):
    """Scalar loop over the allowed keys of each row (no masks, no BLAS)."""
    Lq, Lk = len(q), len(k)
    out, lse = [], []
    for i in range(Lq):
        c = i + Lk - Lq
        js = [j for j in range(Lk)
              if (win[0] < 0 or j >= c - win[0]) and (win[1] < 0 or j <= c + win[1])]
        if not js:
            out.append([0.0] * len(v[0])); lse.append(math.inf); continue
        s = [scale * sum(a * b for a, b in zip(q[i], k[j])) for j in js]
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        tot = sum(w)
        out.append([sum(wi * v[j][col] for wi, j in zip(w, js)) / tot
                    for col in range(len(v[0]))])
        lse.append(mx + math.log(tot))
    return np.array(out), np.array(lse)


@pytest.mark.parametrize("Lq,Lk,win", [(7, 7, (2, 0)), (6, 10, (1, 2)), (10, 6, (0, 1)),
                                       (9, 9, (-1, 3)), (9, 9, (4, -1))])
def test_bruteforce_loops_window(Lq, Lk, win):
    q = rnd((Lq, 3), 13); k = rnd((Lk, 3), 14); v = rnd((Lk, 2), 15)
    o, lse = oracle.attention_forward(q, k, v, 1.1, True, window=win)
    o2, lse2 = _loops_window(q.tolist(), k.tolist(), v.tolist(), 1.1, win)
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, atol=1e-13)


@pytest.mark.parametrize("Lq,Lk,win", [(6, 6, (1, 1)), (4, 7, (2, 0)), (7, 4, (0, 2))])
def test_finite_differences_window(Lq, Lk, win):
    d, scale, eps = 3, 0.9, 1e-6
    q = rnd((Lq, d), 16); k = rnd((Lk, d), 17); v = rnd((Lk, d), 18); do = rnd((Lq, d), 19)

    def loss(qq, kk, vv):
        o, _ = oracle.attention_forward(qq, kk, vv, scale, False, window=win)
        return float((o * do).sum())

    grads = oracle.attention_backward(q, k, v, do, scale, False, window=win)
    base = {"qq": q, "kk": k, "vv": v}
    for name, g in zip(("qq", "kk", "vv"), grads):
        num = np.zeros_like(base[name])
        for idx in np.ndindex(num.shape):
            hi = dict(base); lo = dict(base)
            hi[name] = base[name].copy(); hi[name][idx] += eps
            lo[name] = base[name].copy(); lo[name][idx] -= eps
            num[idx] = (loss(**hi) - loss(**lo)) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-7, err_msg=name)


def test_varlen_window_equals_segments():
    lens_q, lens_k = [5, 1, 12, 7, 3], [5, 4, 12, 2, 0]
    cq = np.concatenate([[0], np.cumsum(lens_q)]); ck = np.concatenate([[0], np.cumsum(lens_k)])
    H, d, win = 2, 4, (2, 1)
    q = rnd((cq[-1], H, d), 20); k = rnd((ck[-1], H, d), 21); v = rnd((ck[-1], H, d), 22)
    do = rnd((cq[-1], H, d), 23)
    o, lse = oracle.varlen_attention_forward(q, k, v, cq, ck, 0.5, True, window=win)
    dq, dk, dv = oracle.varlen_attention_backward(q, k, v, do, cq, ck, 0.5, True, window=win)
    for s in range(len(lens_q)):
        a, b, c, e = cq[s], cq[s + 1], ck[s], ck[s + 1]
        for h in range(H):
            o2, l2 = _loops_window(q[a:b, h].tolist(), k[c:e, h].tolist(), v[c:e, h].tolist(),
                                   0.5, win) if e > c else (np.zeros((b - a, d)),
                                                            np.full(b - a, np.inf))
            if b > a:
                np.testing.assert_allclose(o[a:b, h], o2, atol=1e-13)
                np.testing.assert_allclose(lse[h, a:b], l2, atol=1e-13)
            g = oracle.attention_backward(q[a:b, h], k[c:e, h], v[c:e, h], do[a:b, h], 0.5,
                                          False, window=win)
            np.testing.assert_allclose(dq[a:b, h], g[0], atol=1e-15)
            np.testing.assert_allclose(dk[c:e, h], g[1], atol=1e-15)
            np.testing.assert_allclose(dv[c:e, h], g[2], atol=1e-15)


# ---------------------------------------------------------------- the pins bite
def test_planted_window_mistakes_are_caught(monkeypatch):
    """Mutants of the window mask (sides swapped, right bound off by one, alignment
    top-left instead of bottom-right) must fail the pins above."""
    import oracle.attn_ref as ref
    real = ref.allowed_mask

    def swapped(rows, Lq, Lk, causal, window=None):
        if window is not None:
            window = (window[1], window[0])
        return real(rows, Lq, Lk, causal, window)

    def off_by_one(rows, Lq, Lk, causal, window=None):
        if window is not None and window[1] >= 0:
            window = (window[0], window[1] + 1)
        return real(rows, Lq, Lk, causal, window)

    def top_left(rows, Lq, Lk, causal, window=None):
        return real(np.asarray(rows) - (Lk - Lq), Lq, Lk, causal, window)

    checks = (test_worked_window_left1, test_worked_window_right1,
              test_worked_window_bottom_right_alignment)
    for mutant in (swapped, off_by_one, top_left):
        monkeypatch.setattr(ref, "allowed_mask", mutant)
        caught = 0
        for chk in checks:
            try:
                chk()
            except AssertionError:
                caught += 1
        monkeypatch.setattr(ref, "allowed_mask", real)
        assert caught > 0, mutant.__name__


@pytest.mark.parametrize("Lq,Lk,win", [(50, 50, (7, 0)), (30, 70, (5, 9)), (70, 30, (-1, 4)),
                                       (40, 40, (-1, -1)), (25, 60, (3, -1))])
def test_flop_count_pairs_match_mask(Lq, Lk, win):
    # The workloads' FLOP sizing counts the same pairs the oracle's mask admits.
    from exact_tiled_attention_33_b200 import workloads
    from oracle.attn_ref import allowed_mask
    assert workloads.window_pairs(Lq, Lk, win) == int(allowed_mask(np.arange(Lq), Lq, Lk,
                                                                   False, win).sum())
