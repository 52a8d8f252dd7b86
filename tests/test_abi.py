"""CPU checks of the C ABI boundary: the library loads, exports every entry point the
header declares, and rejects bad arguments on the host (no GPU work is started: every
call here fails validation or is a no-op before any CUDA call)."""

import ctypes
import os
import re

import pytest

from exact_tiled_attention_33_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fattn.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def test_header_declares_expected_calls():
    names = declared_symbols()
    for n in ("fa_fwd", "fa_varlen_fwd", "fa_bwd", "fa_varlen_bwd", "fa_bwd_workspace_size",
              "fa_get_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(declared_symbols()) == set(_lib.SIGNATURES)


def test_status_strings(lib):
    assert lib.fa_status_string(0) == b"ok"
    assert lib.fa_status_string(4) == b"device wait timed out"
    assert lib.fa_status_string(99) == b"unknown status"


def test_workspace_sizes(lib):
    # the backward workspace holds D = rowsum(dO ∘ O) (fp32 [B, H, N]) and the fp32 dQ sums
    # ([rows, H, d]), each rounded up to 256 bytes
    def r256(x):
        return (x + 255) // 256 * 256

    B, N, H, d = 2, 16384, 32, 128
    assert lib.fa_bwd_workspace_size(B, N, H, d) == B * H * N * 4 + B * N * H * d * 4
    assert lib.fa_bwd_workspace_size(1, 3, 1, 64) == 256 + r256(3 * 64 * 4)
    assert lib.fa_bwd_workspace_size(0, 3, 1, 64) == 0
    assert lib.fa_varlen_bwd_workspace_size(896, 32, 128) == 896 * 32 * 4 + 896 * 32 * 128 * 4
    assert lib.fa_varlen_bwd_workspace_size(33, 2, 64) == r256(33 * 2 * 4) + r256(33 * 2 * 64 * 4)


P = ctypes.c_void_p(4096)  # a 16-byte aligned fake address; validation fails before any use


def test_rejects_bad_head_dim(lib):
    assert lib.fa_fwd(P, P, P, P, P, 1, 128, 1, 96, 0.1, 0, 0, None) == _lib.FA_ERR_UNSUPPORTED
    assert b"head_dim" in lib.fa_last_error()


def test_rejects_bad_dtype_and_scale(lib):
    assert lib.fa_fwd(P, P, P, P, P, 1, 128, 1, 64, 0.1, 0, 7, None) == _lib.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd(P, P, P, P, P, 1, 128, 1, 64, float("nan"), 0, 0, None) == \
        _lib.FA_ERR_INVALID_ARG


def test_rejects_null_and_misaligned(lib):
    assert lib.fa_fwd(None, P, P, P, P, 1, 128, 1, 64, 0.1, 0, 0, None) == _lib.FA_ERR_INVALID_ARG
    mis = ctypes.c_void_p(4096 + 8)
    assert lib.fa_fwd(P, mis, P, P, P, 1, 128, 1, 64, 0.1, 0, 0, None) == _lib.FA_ERR_INVALID_ARG
    assert b"aligned" in lib.fa_last_error()


def test_rejects_negative_sizes(lib):
    assert lib.fa_fwd(P, P, P, P, P, -1, 128, 1, 64, 0.1, 0, 0, None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_varlen_fwd(P, P, P, P, P, P, P, 10, 10, 1, 64, 0.1, 0, -2, 10, 10, 0, None) == \
        _lib.FA_ERR_INVALID_ARG
    assert lib.fa_varlen_fwd(P, P, P, P, P, P, P, 20, 10, 1, 64, 0.1, 0, 1, 10, 10, 0, None) == \
        _lib.FA_ERR_INVALID_ARG


def test_size_limits(lib):
    assert lib.fa_fwd(P, P, P, P, P, 70000, 70000, 1, 64, 0.1, 0, 0, None) == \
        _lib.FA_ERR_UNSUPPORTED          # B*N >= 2^31
    assert lib.fa_fwd(P, P, P, P, P, 70000, 16, 1, 64, 0.1, 0, 0, None) == \
        _lib.FA_ERR_UNSUPPORTED          # more batches than a grid dimension holds
    assert lib.fa_bwd(P, P, P, P, P, P, P, P, P, 70000, 16, 1, 64, 0.1, 0, P, 1 << 40, 0,
                      None) == _lib.FA_ERR_UNSUPPORTED


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    # B*H*N above the fixed scratch capacity is refused on the host with a clear message
    st = lib.fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, 8, 16384, 64, 128, 0.1, 1, 0, None)
    assert st == _lib.FA_ERR_UNSUPPORTED
    assert b"scratch capacity" in lib.fa_last_error()
    # the exact edge: B*H*N = 4194305 (= 5 * 838861) is one element over the capacity ...
    assert lib.fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, 1, 838861, 5, 128, 0.1, 1, 0,
                              None) == _lib.FA_ERR_UNSUPPORTED
    assert b"scratch capacity" in lib.fa_last_error()
    # ... while B*H*N = 4194304 passes the capacity check (it then fails later, on this
    # GPU-less host, for a reason that is not the capacity)
    st = lib.fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, 64, 1024, 64, 128, 0.1, 1, 0, None)
    assert st != _lib.FA_OK and b"scratch capacity" not in lib.fa_last_error()


def test_empty_problems_are_noops(lib):
    # zero-size problems return OK without touching (null) pointers or the GPU
    assert lib.fa_fwd(None, None, None, None, None, 0, 128, 1, 64, 0.1, 0, 0, None) == _lib.FA_OK
    assert lib.fa_fwd(None, None, None, None, None, 1, 0, 1, 64, 0.1, 1, 1, None) == _lib.FA_OK
    assert lib.fa_varlen_fwd(None, None, None, None, None, None, None, 0, 0, 1, 64, 0.1, 0, 0, 0,
                             0, 0, None) == _lib.FA_OK


def test_local_window_validation(lib):
    # Windowed calls keep index sums in int32: a bounded window with 2N >= 2^31 is refused
    # on the host before any CUDA call; zero sizes stay no-ops.
    n = 1 << 30
    assert lib.fa_fwd_local(P, P, P, P, P, 1, n, 1, 64, 0.1, 5, 0, 0, None) == \
        _lib.FA_ERR_UNSUPPORTED
    assert b"window" in lib.fa_last_error()
    assert lib.fa_bwd_local(P, P, P, P, P, P, P, P, P, 1, n, 1, 64, 0.1, -1, 7, P, 1 << 40, 0,
                            None) == _lib.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd_local(None, None, None, None, None, 0, 128, 1, 64, 0.1, 3, 3, 0, None) == \
        _lib.FA_OK
    assert lib.fa_varlen_fwd_local(P, P, P, P, P, P, P, 10, 10, 1, 64, 0.1, 4, 4, -2, 10, 10, 0,
                                   None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_varlen_bwd_local(P, P, P, P, P, P, P, P, P, P, P, 10, 10, 1, 96, 0.1, 4, 4, 1,
                                   10, 10, P, 1 << 20, 0, None) == _lib.FA_ERR_UNSUPPORTED


def test_decode_validation(lib):
    # host-side checks of the decode calls (nothing is launched)
    assert lib.fa_decode(P, P, P, P, P, P, 1, 17, 1, 128, 64, 64, 0.1, 1, None, 0, 0, None) == \
        _lib.FA_ERR_UNSUPPORTED                      # Nq > 16
    assert lib.fa_decode(P, P, P, P, P, P, 1, 1, 1, 128, 64, 65, 0.1, 1, None, 0, 0, None) == \
        _lib.FA_ERR_INVALID_ARG                      # max_seqlen_k > capacity
    assert lib.fa_decode(None, None, None, None, None, None, 0, 1, 1, 128, 64, 64, 0.1, 1, None,
                         0, 0, None) == _lib.FA_OK   # B = 0
    assert lib.fa_decode_paged(P, P, P, P, P, P, P, 1, 1, 1, 128, 24, 4, 4, 64, 0.1, 1, None, 0,
                               0, None) == _lib.FA_ERR_UNSUPPORTED   # page size not 2^k
    assert lib.fa_decode_paged(P, P, P, P, P, P, P, 1, 1, 1, 128, 16, 4, 2, 64, 0.1, 1, None, 0,
                               0, None) == _lib.FA_ERR_INVALID_ARG   # 2 blocks x 16 < 64
    # split policy: one split once B*H fills ~8 waves of CTAs, else a workspace for the
    # fp32 partial outputs and log-sum-exps of every split
    assert lib.fa_decode_workspace_size(40, 1, 32, 128, 16384) == 0
    n = lib.fa_decode_workspace_size(8, 1, 32, 128, 16384)
    splits = 5  # ceil(1184 / 256) = 5 splits of ceil(128 / 5) = 26 tiles (5 x 26 >= 128)
    rows = 8 * 1 * 32 * splits
    assert n == -(-rows * 128 * 4 // 256) * 256 + -(-rows * 4 // 256) * 256


def test_fp8_validation(lib):
    # FP8 forward: head_dim 128 only, scale >= 0, descale factors > 0
    assert lib.fa_fwd_fp8(P, P, P, P, P, 1, 128, 1, 64, 0.1, 1.0, 1.0, 1.0, 0, 0, None) == \
        _lib.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd_fp8(P, P, P, P, P, 1, 128, 1, 128, -0.1, 1.0, 1.0, 1.0, 0, 0, None) == \
        _lib.FA_ERR_UNSUPPORTED
    assert lib.fa_fwd_fp8(P, P, P, P, P, 1, 128, 1, 128, 0.1, 0.0, 1.0, 1.0, 0, 0, None) == \
        _lib.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_fp8(None, None, None, None, None, 0, 128, 1, 128, 0.1, 1.0, 1.0, 1.0, 0, 0,
                          None) == _lib.FA_OK
