"""GPU test of the allocation-free backward entry point, fa_bwd_noalloc.

Some callers cannot allocate device memory when they call the library: their device memory
is owned by another allocator (a framework's caching pool that must see every byte), or a
cudaMalloc and its implicit synchronisation is not acceptable inside their loop.
fa_bwd_noalloc serves them: it is fa_bwd with its D scratch in a fixed array inside the
library instead of a caller workspace.

The test calls it through the C ABI twice in a row with different shapes (first a larger
non-causal problem, so that the shared array holds stale values, then a smaller causal one
with another head_dim) and checks each call against fa_bwd_deterministic, the workspace
entry point that runs the same kernels (bitwise equal), and the second call against the
fp64 oracle's analytic gradients on sampled rows, max |dX - dX_ref| <= 2e-2 * max |dX_ref|.
It also checks the capacity edge: B*H*N = 4194304 is accepted (and equals
fa_bwd_deterministic), one more is refused.  The file sorts last so that a run which stops
at its first failure has already run every other test.
"""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_33_b200 import _lib
from exact_tiled_attention_33_b200 import attention as fa
from exact_tiled_attention_33_b200 import workloads as wl
from tests.parity import check_grad, f64

pytestmark = pytest.mark.gpu


def _noalloc(lib, q, k, v, o, lse, do, scale, causal):
    B, N, H, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.current_stream().cuda_stream
    st = lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                            do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                            dv.data_ptr(), B, N, H, d, scale, int(causal), _lib.FA_BF16, stream)
    assert st == _lib.FA_OK, lib.fa_last_error()
    assert lib.fa_get_device_status(stream) == _lib.FA_OK
    return dq, dk, dv


def _inputs(w):
    t = wl.generate(w)
    q, k, v, do = (t[x].to("cuda") for x in ("q", "k", "v", "do"))
    o, lse = fa.fwd(q, k, v, w.softmax_scale, w.causal)
    return t, q, k, v, do, o, lse


def test_noalloc_backward_two_calls_against_workspace_backward_and_oracle():
    lib = _lib.load()
    shapes = [wl.custom("noalloc_big", B=2, N=1500, H=8, d=128, causal=False, seed=31),
              wl.custom("noalloc_small", B=1, N=700, H=4, d=64, causal=True, seed=32)]
    for call, w in enumerate(shapes):
        t, q, k, v, do, o, lse = _inputs(w)
        got = _noalloc(lib, q, k, v, o, lse, do, w.softmax_scale, w.causal)
        ref = fa.bwd(q, k, v, o, lse, do, w.softmax_scale, w.causal, deterministic=True)
        for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
            assert torch.equal(g, r), f"{name} call {call} differs from fa_bwd_deterministic"
    # the second call (after the larger one left its values in the shared array) against
    # the oracle on sampled rows of every head
    qf, kf, vf, dof = (wl.to_f64(t[x]) for x in ("q", "k", "v", "do"))
    dqg, dkg, dvg = (f64(x) for x in got)
    for h in range(w.H):
        rows = wl.sample_rows(w.N, 128, 7000 + h)
        gq, gk, gv = oracle.attention_backward(qf[0, :, h], kf[0, :, h], vf[0, :, h],
                                               dof[0, :, h], w.softmax_scale, w.causal,
                                               dq_rows=rows, dkv_rows=rows)
        check_grad(dqg[0, rows, h], gq, f"noalloc dQ h={h}")
        check_grad(dkg[0, rows, h], gk, f"noalloc dK h={h}")
        check_grad(dvg[0, rows, h], gv, f"noalloc dV h={h}")


def test_noalloc_capacity_edge():
    lib = _lib.load()
    # B*H*N = 64 * 64 * 1024 = 4194304: exactly the capacity, accepted
    w = wl.custom("noalloc_edge", B=64, N=1024, H=64, d=64, causal=True, seed=33)
    t, q, k, v, do, o, lse = _inputs(w)
    got = _noalloc(lib, q, k, v, o, lse, do, w.softmax_scale, True)
    ref = fa.bwd(q, k, v, o, lse, do, w.softmax_scale, True, deterministic=True)
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        assert torch.equal(g, r), f"{name} at the capacity edge differs from fa_bwd_deterministic"
    qf, kf, vf, dof = (wl.to_f64(t[x]) for x in ("q", "k", "v", "do"))
    for (b, h) in [(0, 0), (63, 63)]:  # the first and the last D slot of the array
        gq, gk, gv = oracle.attention_backward(qf[b, :, h], kf[b, :, h], vf[b, :, h],
                                               dof[b, :, h], w.softmax_scale, True)
        for name, g, r in zip(("dQ", "dK", "dV"), got, (gq, gk, gv)):
            check_grad(f64(g)[b, :, h], r, f"noalloc edge {name}[{b},{h}]")
    # one element more is refused on the host, before anything is launched
    P = q.data_ptr()
    st = lib.fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, 1, 838861, 5, 128, 0.1, 1,
                            _lib.FA_BF16, None)
    assert st == _lib.FA_ERR_UNSUPPORTED and b"scratch capacity" in lib.fa_last_error()
    assert np.isfinite(f64(got[0])).all()
