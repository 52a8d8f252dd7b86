"""The O(N) memory claim of the pages (the N x N score matrix is never stored): a forward
and backward through the C ABI with every buffer allocated by the caller leave the device's
free memory unchanged — the library allocates nothing, let alone anything proportional to
N^2 (at the size below one N x N fp32 score matrix per head would take 8.6 GB)."""

import pytest
import torch

from exact_tiled_attention_33_b200 import _lib
from exact_tiled_attention_33_b200 import attention as fa

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_no_device_allocation_in_forward_and_backward():
    B, N, H, d = 1, 16384, 8, 128
    g = torch.Generator(device="cpu").manual_seed(21)
    q, k, v, do = (torch.randn((B, N, H, d), generator=g).to(torch.bfloat16).to(DEV)
                   for _ in range(4))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=DEV)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = fa.bwd_workspace(B, N, H, d, q.device)
    # the backward's workspace is linear in N: D (B*H*N floats) and the fp32 dQ sums
    # (B*N*H*d floats), never an N x N buffer
    assert ws.numel() == B * H * N * 4 + B * N * H * d * 4
    lib = _lib.load()
    st = torch.cuda.current_stream().cuda_stream
    scale = d ** -0.5

    def call():
        assert lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                          lse.data_ptr(), B, N, H, d, scale, 1, _lib.FA_BF16, st) == 0
        assert lib.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                          do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                          dv.data_ptr(), B, N, H, d, scale, 1, ws.data_ptr(), ws.numel(),
                          _lib.FA_BF16, st) == 0

    call()  # first launches load the kernels
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    assert fa.device_status() == 0
