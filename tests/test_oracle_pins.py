"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test checks the oracle against something the pages or the mathematics fix: a
hand-worked closed form, an invariant of softmax attention, a brute-force scalar
loop, central finite differences, the pages' online-softmax merge rule (page
"FlashAttention实战：如何在A100上实现3倍加速的Transformer训练" §3.1), a library
autograd witness on tiny inputs, and the shapes the pages print.  The set is chosen so
that a dropped term, a wrong sign, a wrong index or a transposed operand in the oracle
fails at least one test (see test_planted_mistakes_are_caught).
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_33_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LN3, LN4, LN8 = math.log(3.0), math.log(4.0), math.log(8.0)


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- hand-worked cases
# d = 1, scale = 1, q = 1 and keys chosen so the scores are logs of small integers:
# exp(scores) are then integers and every softmax weight, output and gradient is a
# short closed form worked out by hand (below each case).

def test_worked_example_noncausal():
    # scores [0, ln3] -> weights [1/4, 3/4]; O = 4/4 + 3*8/4 = 7; LSE = ln(1+3).
    # dO = 1: D = 7; dP = [4, 8]; dS = [1/4(4-7), 3/4(8-7)] = [-3/4, 3/4]
    # dQ = -3/4*0 + 3/4*ln3; dK = dS * q = [-3/4, 3/4]; dV = weights.
    q = np.array([[1.0]]); k = np.array([[0.0], [LN3]]); v = np.array([[4.0], [8.0]])
    o, lse = oracle.attention_forward(q, k, v, 1.0, False)
    assert o[0, 0] == pytest.approx(7.0, abs=1e-14)
    assert lse[0] == pytest.approx(LN4, abs=1e-14)
    dq, dk, dv = oracle.attention_backward(q, k, v, np.ones((1, 1)), 1.0, False)
    assert dq[0, 0] == pytest.approx(0.75 * LN3, abs=1e-14)
    np.testing.assert_allclose(dk[:, 0], [-0.75, 0.75], atol=1e-14)
    np.testing.assert_allclose(dv[:, 0], [0.25, 0.75], atol=1e-14)


def test_worked_example_causal_square():
    # Lq = Lk = 2, causal.  Row 0 sees key 0 only: O0 = 4, LSE0 = 0, dS0 = [1*(4-4), 0].
    # Row 1 as in the non-causal case.  dV = [1 + 1/4, 3/4]; dK = [-3/4, 3/4].
    q = np.array([[1.0], [1.0]]); k = np.array([[0.0], [LN3]]); v = np.array([[4.0], [8.0]])
    o, lse = oracle.attention_forward(q, k, v, 1.0, True)
    np.testing.assert_allclose(o[:, 0], [4.0, 7.0], atol=1e-14)
    np.testing.assert_allclose(lse, [0.0, LN4], atol=1e-14)
    dq, dk, dv = oracle.attention_backward(q, k, v, np.ones((2, 1)), 1.0, True)
    np.testing.assert_allclose(dq[:, 0], [0.0, 0.75 * LN3], atol=1e-14)
    np.testing.assert_allclose(dk[:, 0], [-0.75, 0.75], atol=1e-14)
    np.testing.assert_allclose(dv[:, 0], [1.25, 0.75], atol=1e-14)


def test_worked_example_causal_bottom_right():
    # Lq = 2 < Lk = 3: key j allowed for row i iff j <= i + 1.
    # Row 0 sees keys {0,1}: weights [1/4, 3/4, 0], O0 = 7, LSE0 = ln4.
    # Row 1 sees keys {0,1,2}: exp(scores) = [1, 3, 4] -> weights [1/8, 3/8, 1/2],
    #   O1 = 4/8 + 24/8 + 0 = 3.5, LSE1 = ln8.
    # dO = 1: dV = [1/4+1/8, 3/4+3/8, 1/2]
    #   dS0 = [-3/4, 3/4, 0];  dS1 = [1/8(4-3.5), 3/8(8-3.5), 1/2(0-3.5)]
    #   dQ0 = 3/4 ln3;  dQ1 = 27/16 ln3 - 7/4 ln4;  dK = dS0 + dS1.
    q = np.array([[1.0], [1.0]])
    k = np.array([[0.0], [LN3], [LN4]])
    v = np.array([[4.0], [8.0], [0.0]])
    o, lse = oracle.attention_forward(q, k, v, 1.0, True)
    np.testing.assert_allclose(o[:, 0], [7.0, 3.5], atol=1e-14)
    np.testing.assert_allclose(lse, [LN4, LN8], atol=1e-14)
    dq, dk, dv = oracle.attention_backward(q, k, v, np.ones((2, 1)), 1.0, True)
    np.testing.assert_allclose(dv[:, 0], [0.375, 1.125, 0.5], atol=1e-14)
    np.testing.assert_allclose(dq[:, 0], [0.75 * LN3, 1.6875 * LN3 - 1.75 * LN4], atol=1e-13)
    np.testing.assert_allclose(dk[:, 0], [-0.6875, 2.4375, -1.75], atol=1e-14)


def test_fully_masked_rows():
    # Lq = 3 > Lk = 1 causal: rows 0 and 1 see no key (j <= i - 2); row 2 sees key 0.
    q = rnd((3, 4), 1); k = rnd((1, 4), 2); v = rnd((1, 4), 3); do = rnd((3, 4), 4)
    o, lse = oracle.attention_forward(q, k, v, 0.5, True)
    assert np.all(o[:2] == 0.0) and np.all(np.isposinf(lse[:2]))
    np.testing.assert_allclose(o[2], v[0], atol=1e-15)
    assert lse[2] == pytest.approx(0.5 * q[2] @ k[0], abs=1e-14)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.5, True)
    assert np.all(dq[:2] == 0.0)
    # Single allowed key: the weight is exactly 1, so dS = 1*(dP - D) = 0.
    np.testing.assert_allclose(dq[2], 0.0, atol=1e-14)
    np.testing.assert_allclose(dk, 0.0, atol=1e-14)
    np.testing.assert_allclose(dv[0], do[2], atol=1e-15)


def test_zero_keys():
    q = rnd((4, 8), 5)
    o, lse = oracle.attention_forward(q, np.zeros((0, 8)), np.zeros((0, 8)), 0.3, False)
    assert o.shape == (4, 8) and np.all(o == 0) and np.all(np.isposinf(lse))


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("causal", [False, True])
def test_rows_sum_to_one(causal):  # P1
    q = rnd((37, 16), 10); k = rnd((37, 16), 11)
    p = oracle.softmax_probs(q, k, 0.25, causal)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)
    assert np.all(p >= 0)
    if causal:
        assert np.all(np.triu(p, 1) == 0.0)


def test_single_key_returns_v():  # P2
    q = rnd((9, 16), 12); k = rnd((1, 16), 13); v = rnd((1, 16), 14)
    o, lse = oracle.attention_forward(q, k, v, 0.7, False)
    np.testing.assert_allclose(o, np.repeat(v, 9, axis=0), atol=1e-15)
    np.testing.assert_allclose(lse, 0.7 * (q @ k[0]), atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_returns_v(causal):  # P3
    q = rnd((33, 8), 15); k = rnd((33, 8), 16)
    vrow = rnd((1, 8), 17)
    o, _ = oracle.attention_forward(q, k, np.repeat(vrow, 33, axis=0), 0.9, causal)
    np.testing.assert_allclose(o, np.repeat(vrow, 33, axis=0), atol=1e-13)


def test_causal_row0_is_v0():  # P4
    q = rnd((20, 8), 18); k = rnd((20, 8), 19); v = rnd((20, 8), 20)
    o, lse = oracle.attention_forward(q, k, v, 0.4, True)
    np.testing.assert_allclose(o[0], v[0], atol=1e-15)
    assert lse[0] == pytest.approx(0.4 * q[0] @ k[0], abs=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_scale_zero_closed_form(causal):  # P6
    q = rnd((24, 8), 21); k = rnd((24, 8), 22); v = rnd((24, 8), 23)
    o, lse = oracle.attention_forward(q, k, v, 0.0, causal)
    for i in range(24):
        n = i + 1 if causal else 24
        np.testing.assert_allclose(o[i], v[:n].mean(axis=0), atol=1e-14)
        assert lse[i] == pytest.approx(math.log(n), abs=1e-14)


def test_key_permutation_and_shift():  # P7
    q = rnd((16, 8), 24); k = rnd((29, 8), 25); v = rnd((29, 8), 26)
    o, lse = oracle.attention_forward(q, k, v, 0.6, False)
    perm = np.random.default_rng(27).permutation(29)
    o2, lse2 = oracle.attention_forward(q, k[perm], v[perm], 0.6, False)
    np.testing.assert_allclose(o2, o, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, atol=1e-13)
    u = rnd((1, 8), 28)
    o3, lse3 = oracle.attention_forward(q, k + u, v, 0.6, False)
    np.testing.assert_allclose(o3, o, atol=1e-12)
    np.testing.assert_allclose(lse3, lse + 0.6 * (q @ u[0]), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_invariants(causal):  # P8
    L, d = 21, 8
    q = rnd((L, d), 30); k = rnd((L, d), 31); v = rnd((L, d), 32); do = rnd((L, d), 33)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.45, causal)
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-12)        # rows of dS sum to 0
    np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), atol=1e-12)  # rows of P sum to 1
    kc = np.repeat(rnd((1, d), 34), L, axis=0)
    dqc, _, _ = oracle.attention_backward(q, kc, v, do, 0.45, causal)
    np.testing.assert_allclose(dqc, 0.0, atol=1e-12)                    # constant K
    ones = np.ones((L, d))
    _, _, dv1 = oracle.attention_backward(q, k, v, ones, 0.45, causal)  # loss = output.sum()
    p = oracle.softmax_probs(q, k, 0.45, causal)
    np.testing.assert_allclose(dv1, np.repeat(p.sum(axis=0)[:, None], d, axis=1), atol=1e-13)


# ---------------------------------------------------------------- brute force
def _loops_forward(q, k, v, scale, causal):
    """Scalar triple loop, no BLAS: a second, independent writing of the definition."""
    Lq, d = len(q), len(q[0])
    Lk = len(k)
    out, lse = [], []
    for i in range(Lq):
        s = []
        for j in range(Lk):
            if causal and j > i + (Lk - Lq):
                continue
            acc = 0.0
            for c in range(d):
                acc += q[i][c] * k[j][c]
            s.append((j, scale * acc))
        if not s:
            out.append([0.0] * len(v[0])); lse.append(math.inf); continue
        mx = max(x for _, x in s)
        w = [(j, math.exp(x - mx)) for j, x in s]
        tot = sum(x for _, x in w)
        out.append([sum(x * v[j][c] for j, x in w) / tot for c in range(len(v[0]))])
        lse.append(mx + math.log(tot))
    return np.array(out), np.array(lse)


@pytest.mark.parametrize("Lq,Lk,causal", [(7, 7, False), (7, 7, True), (5, 9, True),
                                          (9, 5, True), (16, 11, False)])
def test_bruteforce_loops(Lq, Lk, causal):  # P9 (forward)
    q = rnd((Lq, 4), 40); k = rnd((Lk, 4), 41); v = rnd((Lk, 3), 42)
    o, lse = oracle.attention_forward(q, k, v, 0.8, causal)
    o2, lse2 = _loops_forward(q.tolist(), k.tolist(), v.tolist(), 0.8, causal)
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, atol=1e-13)


@pytest.mark.parametrize("Lq,Lk,causal", [(6, 6, False), (6, 6, True), (4, 7, True)])
def test_finite_differences(Lq, Lk, causal):  # P9 (backward)
    d, scale, eps = 3, 0.9, 1e-6
    q = rnd((Lq, d), 50); k = rnd((Lk, d), 51); v = rnd((Lk, d), 52); do = rnd((Lq, d), 53)

    def loss(qq, kk, vv):
        o, _ = oracle.attention_forward(qq, kk, vv, scale, causal)
        return float((o * do).sum())

    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale, causal)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}; args_p[name] = xp
            args_m = {"q": q, "k": k, "v": v}; args_m[name] = xm
            num[idx] = (loss(**{"qq": args_p["q"], "kk": args_p["k"], "vv": args_p["v"]})
                        - loss(**{"qq": args_m["q"], "kk": args_m["k"], "vv": args_m["v"]})) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-7, err_msg=f"d{name}")


@pytest.mark.parametrize("causal", [False, True])
def test_torch_autograd_witness(causal):  # P10: a library routine used as a witness only
    L, d, scale = 13, 8, 0.35
    q = rnd((L, d), 60); k = rnd((L, d), 61); v = rnd((L, d), 62); do = rnd((L, d), 63)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    s = scale * tq @ tk.T
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(L, L, dtype=torch.bool), 1), float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    (o * torch.tensor(do)).sum().backward()
    o_ref, lse_ref = oracle.attention_forward(q, k, v, scale, causal)
    np.testing.assert_allclose(o_ref, o.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(lse_ref, torch.logsumexp(s, -1).detach().numpy(), atol=1e-12)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale, causal)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-12)


# ---------------------------------------------------------------- the pages' merge rule
def _online(q, k, v, scale, causal, chunks):
    """Streaming evaluation with the pages' running statistics (max m, rescaled sum l),
    extended to the output accumulator with the same rescale factor."""
    Lq, Lk = q.shape[0], k.shape[0]
    O = np.zeros((Lq, v.shape[1])); m = np.full(Lq, -np.inf); l = np.zeros(Lq)
    for a, b in chunks:
        s = scale * q @ k[a:b].T
        if causal:
            j = np.arange(a, b)
            s = np.where(j[None, :] <= np.arange(Lq)[:, None] + (Lk - Lq), s, -np.inf)
        m_cur = s.max(axis=1)
        m_new = np.maximum(m, m_cur)
        safe = np.where(np.isfinite(m_new), m_new, 0.0)
        alpha = np.exp(np.where(np.isfinite(m), m - safe, -np.inf))
        p = np.exp(s - safe[:, None])
        l = alpha * l + p.sum(axis=1)
        O = alpha[:, None] * O + p @ v[a:b]
        m = m_new
    return O / l[:, None], m + np.log(l)


@pytest.mark.parametrize("causal", [False, True])
def test_online_merge_equals_two_pass(causal):  # P5
    L, d = 50, 8
    q = 3 * rnd((L, d), 70); k = rnd((L, d), 71); v = rnd((L, d), 72)
    rng = np.random.default_rng(73)
    for _ in range(5):
        cuts = sorted(set(rng.integers(1, L, size=6).tolist()))
        bounds = list(zip([0] + cuts, cuts + [L]))
        o1, lse1 = _online(q, k, v, 0.5, causal, bounds)
        o2, lse2 = oracle.attention_forward(q, k, v, 0.5, causal)
        np.testing.assert_allclose(o1, o2, atol=1e-13)
        np.testing.assert_allclose(lse1, lse2, atol=1e-13)


def test_pages_merge_rule_statistics():
    # The page's two-statistic merge: l = e^(m_prev - m) l_prev + e^(m_cur - m) l_cur.
    x = rnd(40, 74) * 4
    a, b = x[:17], x[17:]
    m_prev, l_prev = a.max(), np.exp(a - a.max()).sum()
    m_cur, l_cur = b.max(), np.exp(b - b.max()).sum()
    m = max(m_prev, m_cur)
    l = math.exp(m_prev - m) * l_prev + math.exp(m_cur - m) * l_cur
    # The oracle's LSE of the concatenated row equals m + ln l.
    q = np.ones((1, 1)); k = x[:, None]
    _, lse = oracle.attention_forward(q, k, np.zeros((40, 1)), 1.0, False)
    assert lse[0] == pytest.approx(m + math.log(l), abs=1e-13)


# ---------------------------------------------------------------- varlen, batching, sampling
def test_varlen_equals_segments():  # P11
    lens = [5, 1, 12, 7]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, d = cu[-1], 2, 4
    q = rnd((T, H, d), 80); k = rnd((T, H, d), 81); v = rnd((T, H, d), 82); do = rnd((T, H, d), 83)
    o, lse = oracle.varlen_attention_forward(q, k, v, cu, cu, 0.5, True)
    dq, dk, dv = oracle.varlen_attention_backward(q, k, v, do, cu, cu, 0.5, True)
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        for h in range(H):
            o2, l2 = oracle.attention_forward(q[a:b, h], k[a:b, h], v[a:b, h], 0.5, True)
            np.testing.assert_allclose(o[a:b, h], o2, atol=1e-15)
            np.testing.assert_allclose(lse[h, a:b], l2, atol=1e-15)
            g = oracle.attention_backward(q[a:b, h], k[a:b, h], v[a:b, h], do[a:b, h], 0.5, True)
            np.testing.assert_allclose(dq[a:b, h], g[0], atol=1e-15)
            np.testing.assert_allclose(dk[a:b, h], g[1], atol=1e-15)
            np.testing.assert_allclose(dv[a:b, h], g[2], atol=1e-15)
    # Segment isolation: changing another segment's keys changes nothing here.
    k2 = k.copy(); k2[cu[2]:cu[3]] += 5.0
    o3, _ = oracle.varlen_attention_forward(q, k2, v, cu, cu, 0.5, True)
    np.testing.assert_array_equal(o3[:cu[2]], o[:cu[2]])


def test_batched_layout():
    B, N, H, d = 2, 9, 3, 4
    q = rnd((B, N, H, d), 90); k = rnd((B, N, H, d), 91); v = rnd((B, N, H, d), 92)
    o, lse = oracle.attention_forward_bhsd(q, k, v, 0.5, True)
    assert o.shape == (B, N, H, d) and lse.shape == (B, H, N)
    o1, l1 = oracle.attention_forward(q[1, :, 2], k[1, :, 2], v[1, :, 2], 0.5, True)
    np.testing.assert_allclose(o[1, :, 2], o1, atol=1e-15)
    np.testing.assert_allclose(lse[1, 2], l1, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_batched_backward_layout(causal):
    # attention_backward_bhsd on the [batch, seqlen, heads, head_dim] layout against torch
    # autograd of the naive formula evaluated directly on that layout (a library witness,
    # independent of the oracle): B != H and unequal sizes make a swapped batch/head or
    # seqlen/head index, or a gradient written to the wrong slot, fail.
    B, N, H, d, scale = 2, 7, 3, 4, 0.6
    q = rnd((B, N, H, d), 97); k = rnd((B, N, H, d), 98); v = rnd((B, N, H, d), 99)
    do = rnd((B, N, H, d), 100)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    s = scale * torch.einsum("bihc,bjhc->bhij", tq, tk)
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    o = torch.einsum("bhij,bjhc->bihc", torch.softmax(s, dim=-1), tv)
    (o * torch.tensor(do)).sum().backward()
    dq, dk, dv = oracle.attention_backward_bhsd(q, k, v, do, scale, causal)
    assert dq.shape == q.shape and dk.shape == k.shape and dv.shape == v.shape
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-12)


def test_row_subsets_match_full():
    L, d = 2100, 16  # spans more than two oracle row blocks
    q = rnd((L, d), 93); k = rnd((L, d), 94); v = rnd((L, d), 95); do = rnd((L, d), 96)
    rows = workloads.sample_rows(L, 40, 7)
    o_full, lse_full = oracle.attention_forward(q, k, v, 0.25, True)
    o_s, lse_s = oracle.attention_forward(q, k, v, 0.25, True, rows=rows)
    np.testing.assert_allclose(o_s, o_full[rows], atol=1e-14)
    np.testing.assert_allclose(lse_s, lse_full[rows], atol=1e-14)
    dq_f, dk_f, dv_f = oracle.attention_backward(q[:300], k[:300], v[:300], do[:300], 0.25, True)
    r = np.array([0, 1, 127, 128, 299])
    dq_s, dk_s, dv_s = oracle.attention_backward(q[:300], k[:300], v[:300], do[:300], 0.25, True,
                                                 dq_rows=r, dkv_rows=r)
    np.testing.assert_allclose(dq_s, dq_f[r], atol=1e-13)
    np.testing.assert_allclose(dk_s, dk_f[r], atol=1e-13)
    np.testing.assert_allclose(dv_s, dv_f[r], atol=1e-13)


def test_pages_printed_examples():  # P12
    g = json.load(open(os.path.join(GOLDEN, "pages_examples.json")))
    ex = g["varlen_example"]
    w = workloads.get("varlen3")
    assert list(w.seqlens) == ex["seqlens"] and w.total == ex["total"]
    assert w.cu_seqlens().tolist() == ex["cu_seqlens"] and max(w.seqlens) == ex["max_seqlen"]
    t = workloads.generate(w)
    cu = t["cu_seqlens"].numpy()
    o, lse = oracle.varlen_attention_forward(workloads.to_f64(t["q"]), workloads.to_f64(t["k"]),
                                             workloads.to_f64(t["v"]), cu, cu,
                                             w.softmax_scale, ex["causal"])
    assert list(o.shape) == ex["output_shape"] and lse.shape == (ex["heads"], ex["total"])
    dense = g["dense_causal_example"]
    assert list(workloads.get("llama_causal").shape()) == dense["output_shape"]


# ---------------------------------------------------------------- the pins bite
def test_planted_mistakes_are_caught(monkeypatch):
    """Mutants of the oracle's backward (dropped scale, wrong sign, transposed product)
    must fail the finite-difference or worked-example pins."""
    import oracle.attn_ref as ref
    real = ref.attention_backward

    def dropped_scale(*a, **kw):
        dq, dk, dv = real(*a, **kw)
        return dq / a[4] if a[4] else dq, dk, dv

    def wrong_sign(*a, **kw):
        dq, dk, dv = real(*a, **kw)
        return dq, -dk, dv

    for mutant in (dropped_scale, wrong_sign):
        monkeypatch.setattr(oracle, "attention_backward", mutant)
        with pytest.raises(AssertionError):
            test_finite_differences(6, 6, True)
        monkeypatch.setattr(oracle, "attention_backward", real)

    real_fwd = ref.attention_forward

    def off_by_one_causal(q, k, v, scale, causal, rows=None):
        if causal:  # shifts the diagonal by one key
            k = np.concatenate([k[1:], k[:1]]) if len(k) > 1 else k
        return real_fwd(q, k, v, scale, causal, rows)

    monkeypatch.setattr(oracle, "attention_forward", off_by_one_causal)
    with pytest.raises(AssertionError):
        test_causal_row0_is_v0()
    monkeypatch.setattr(oracle, "attention_forward", real_fwd)
