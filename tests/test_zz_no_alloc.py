"""GPU test of the allocation-free backward entry point, fa_bwd_noalloc.

Some callers cannot allocate device memory when they call the library (their device
memory is owned by another allocator, or a cudaMalloc and its implicit synchronisation is
not acceptable in their loop).  fa_bwd_noalloc serves them: it is fa_bwd with its D
scratch in a fixed array inside the library instead of a caller workspace.  This test
calls it twice in a row through the C ABI and checks each result against fa_bwd (the
workspace entry point) with the gradient tolerance the parity tests use, max |dX - dX_ref|
<= 2e-2 * max |dX_ref|; the two paths run the same kernels on the same inputs, so the
results are also expected to be bitwise equal.  The file sorts last so that a run which
stops at its first failure has already run every other test.
"""

import pytest
import torch

from exact_tiled_attention_33_b200 import _lib
from exact_tiled_attention_33_b200 import attention as fa
from exact_tiled_attention_33_b200 import workloads as wl
from tests.parity import check_grad, f64

pytestmark = pytest.mark.gpu


def test_noalloc_backward_matches_workspace_backward_twice():
    lib = _lib.load()
    w = wl.custom("noalloc", B=2, N=700, H=4, d=128, causal=True, seed=31)
    t = wl.generate(w)
    q, k, v, do = (t[x].to("cuda") for x in ("q", "k", "v", "do"))
    B, N, H, d = q.shape
    o, lse = fa.fwd(q, k, v, w.softmax_scale, w.causal)
    ref = fa.bwd(q, k, v, o, lse, do, w.softmax_scale, w.causal)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        st = lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                dv.data_ptr(), B, N, H, d, w.softmax_scale, int(w.causal),
                                _lib.FA_BF16, stream)
        assert st == _lib.FA_OK, lib.fa_last_error()
        assert lib.fa_get_device_status(stream) == _lib.FA_OK
        for name, got, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref):
            check_grad(f64(got), f64(r), f"{name} call {call}")
            assert torch.equal(got, r), f"{name} call {call} differs from fa_bwd"
