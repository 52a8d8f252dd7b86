"""GPU parity at the size limits the C ABI accepts: the largest batch (B = 65535, the grid's
z extent) and head count (H = 65535, its y extent), and one 131072-token sequence (1024
query tiles, each walking up to 1024 key tiles), forward and backward through the C ABI
against the fp64 oracle on sampled outputs.

At N = 131072 the oracle's dK/dV of an arbitrary key needs every query row; the sampled key
rows are taken among the last 512 positions, whose only causal queries are the last 512
rows, so the oracle runs on that query block against all keys (bottom-right alignment keeps
each row's position) and gives those keys' exact gradients."""

import numpy as np
import pytest

import oracle
from exact_tiled_attention_33_b200 import attention as fa
from exact_tiled_attention_33_b200 import workloads as wl
from tests.parity import check_grad, check_lse, check_o, f64
from tests.test_bwd_gpu import run_dense_bwd
from tests.test_fwd_gpu import run_dense

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("causal", [False, True])
def test_largest_batch(causal):
    w = wl.custom("limit_batch", B=65535, N=3, H=1, d=64, causal=causal, seed=72)
    pairs = [(0, 0), (1, 0), (32767, 0), (65534, 0)]
    run_dense(w, bh_subset=pairs)
    run_dense_bwd(w, dq_heads=pairs, dkv_heads=pairs)


@pytest.mark.parametrize("causal", [False, True])
def test_most_heads(causal):
    w = wl.custom("limit_heads", B=1, N=3, H=65535, d=64, causal=causal, seed=73)
    pairs = [(0, 0), (0, 1), (0, 40000), (0, 65534)]
    run_dense(w, bh_subset=pairs)
    run_dense_bwd(w, dq_heads=pairs, dkv_heads=pairs)


def test_longest_sequence_131072():
    N, tail = 131072, 512
    w = wl.custom("limit_long", B=1, N=N, H=1, d=64, causal=True, seed=71)
    run_dense(w, rows_per_head=48)                       # O and LSE on sampled rows
    t = wl.generate(w)
    q, k, v, do = (t[x].to(DEV) for x in ("q", "k", "v", "do"))
    o, lse = fa.fwd(q, k, v, w.softmax_scale, True)
    dq, dk, dv = fa.bwd(q, k, v, o, lse, do, w.softmax_scale, True)
    assert fa.device_status() == 0
    qf, kf, vf, dof = (wl.to_f64(t[x])[0, :, 0] for x in ("q", "k", "v", "do"))
    none = np.zeros(0, np.int64)
    rows = wl.sample_rows(N, 32, 5000)
    gq_ref, _, _ = oracle.attention_backward(qf, kf, vf, dof, w.softmax_scale, True,
                                             dq_rows=rows, dkv_rows=none)
    check_grad(f64(dq)[0, rows, 0], gq_ref, "dQ sampled rows")
    keys = np.unique(np.concatenate([np.arange(N - 8, N),
                                     np.random.default_rng(5001).choice(
                                         np.arange(N - tail, N - 8), 24, replace=False)]))
    _, gk_ref, gv_ref = oracle.attention_backward(qf[N - tail:], kf, vf, dof[N - tail:],
                                                  w.softmax_scale, True, dq_rows=none,
                                                  dkv_rows=keys)
    check_grad(f64(dk)[0, keys, 0], gk_ref, "dK of the last keys")
    check_grad(f64(dv)[0, keys, 0], gv_ref, "dV of the last keys")
