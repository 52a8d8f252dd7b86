"""CPU test of the kernels' tile scheduling: `key_tile_range` (which K/V tiles a query tile
walks: forward and dQ pass) and `query_tile_range` (which query tiles a key tile walks: dK/dV
pass), compiled for the host from the library's own header.  For every small shape, window
and tile size, the tiles returned must be exactly the tiles that hold at least one allowed
(query, key) pair of the oracle's mask: none missed (that would drop keys) and none extra
(wasted work).  Tile sizes below 128 exercise many more tile boundaries than the kernels'
128 while running the same arithmetic."""

import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from exact_tiled_attention_33_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_tiled_attention_33_b200", "csrc")
WINDOWS = [(-1, -1), (-1, 0), (0, 0), (0, -1), (1, 0), (2, 3), (5, 0), (0, 4), (-1, 2), (3, -1)]


def _nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.fixture(scope="module")
def shim(tmp_path_factory):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not found")
    out = tmp_path_factory.mktemp("shim") / "libtile_range_shim.so"
    cmd = [nvcc, "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-I", CSRC,
           "-gencode", "arch=compute_100a,code=sm_100a",
           os.path.join(ROOT, "tests", "c", "tile_range_shim.cu"), "-o", str(out)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    lib = ctypes.CDLL(str(out))
    for f in (lib.shim_key_tile_range, lib.shim_query_tile_range):
        f.argtypes = [ctypes.c_int] * 7 + [ctypes.POINTER(ctypes.c_int)] * 2
        f.restype = None
    return lib


def _call(f, a0, a1, L, diag, wl, wr, T):
    b, c = ctypes.c_int(-7), ctypes.c_int(-7)
    f(a0, a1, L, diag, wl, wr, T, ctypes.byref(b), ctypes.byref(c))
    assert c.value >= 0
    return set(range(b.value, b.value + c.value))


@pytest.mark.parametrize("T", [1, 2, 3, 4, 128])
def test_tile_ranges_match_the_mask(shim, T):
    checked = 0
    for Lq in range(1, 10):
        for Lk in range(1, 10):
            diag = Lk - Lq
            for win in WINDOWS:
                mask = oracle.allowed_mask(np.arange(Lq), Lq, Lk, False, window=win)
                for q0 in range(0, Lq, T):      # query tiles, as the forward and dQ pass cut them
                    q1 = min(q0 + T, Lq) - 1
                    want = {int(j) // T for j in np.nonzero(mask[q0:q1 + 1].any(axis=0))[0]}
                    got = _call(shim.shim_key_tile_range, q0, q1, Lk, diag, *win, T)
                    assert got == want, (Lq, Lk, win, T, q0, got, want)
                    checked += 1
                for k0 in range(0, Lk, T):      # key tiles, as the dK/dV pass cuts them
                    k1 = min(k0 + T, Lk) - 1
                    want = {int(i) // T for i in np.nonzero(mask[:, k0:k1 + 1].any(axis=1))[0]}
                    got = _call(shim.shim_query_tile_range, k0, k1, Lq, diag, *win, T)
                    assert got == want, (Lq, Lk, win, T, k0, got, want)
                    checked += 1
    assert checked > 0


def test_tile_ranges_at_kernel_sizes(shim):
    # the kernels' 128-row tiles on the pages' shapes (16K causal, a 4096-key window, a
    # decode-like 4 rows over 8192 keys, Lq != Lk with a two-sided window): sampled tiles of
    # both kinds against the oracle's mask of those rows / keys
    T = 128
    for Lq, Lk, win in ((16384, 16384, (-1, 0)), (16384, 16384, (4096, 0)), (4, 8192, (-1, 0)),
                        (1000, 3000, (100, 100))):
        diag = Lk - Lq
        nq, nk = (Lq + T - 1) // T, (Lk + T - 1) // T
        for t in sorted({0, 1, nq // 3, nq // 2, nq - 2, nq - 1} & set(range(nq))):
            q0, q1 = t * T, min(t * T + T, Lq) - 1
            m = oracle.allowed_mask(np.arange(q0, q1 + 1), Lq, Lk, False, window=win)
            want = {int(j) // T for j in np.nonzero(m.any(axis=0))[0]}
            assert _call(shim.shim_key_tile_range, q0, q1, Lk, diag, *win, T) == want
        full = oracle.allowed_mask(np.arange(Lq), Lq, Lk, False, window=win)
        for t in sorted({0, 1, nk // 3, nk // 2, nk - 2, nk - 1} & set(range(nk))):
            k0, k1 = t * T, min(t * T + T, Lk) - 1
            want = {int(i) // T for i in np.nonzero(full[:, k0:k1 + 1].any(axis=1))[0]}
            assert _call(shim.shim_query_tile_range, k0, k1, Lq, diag, *win, T) == want



def _grid_item(shim, L, T, H, HB, group):
    f = shim.shim_grouped_grid_item
    f.argtypes = [ctypes.c_ulonglong] * 5 + [ctypes.POINTER(ctypes.c_int)]
    f.restype = None
    out = (ctypes.c_int * 3)(-1, -1, -1)
    f(L, T, H, HB, group, out)
    return tuple(out)


@pytest.mark.parametrize("T,H,B,group", [(1, 1, 1, 4), (3, 2, 1, 4), (5, 3, 3, 4), (4, 7, 2, 2),
                                         (2, 5, 1, 1), (128, 32, 2, 4), (8, 16, 8, 4),
                                         (6, 1, 9, 4)])
def test_launch_order_is_a_grouped_tile_major_bijection(shim, T, H, B, group):
    """The forward and the fused backward map a CTA's linear launch index to (tile, head,
    batch) with `grouped_grid_item`: every work item exactly once; groups of `group`
    consecutive (batch, head) pairs (the last one possibly smaller) one after the other; and
    inside a group tile 0 of each of its pairs first, then tile 1, and so on."""
    HB = H * B
    items = [_grid_item(shim, L, T, H, HB, group) for L in range(T * HB)]
    # the 32-bit arithmetic the kernels take for grids below 2^32 CTAs agrees with 64 bits
    f = shim.shim_grouped_grid_item_u64
    f.argtypes = [ctypes.c_ulonglong] * 5 + [ctypes.POINTER(ctypes.c_int)]
    f.restype = None
    for L in range(T * HB):
        out = (ctypes.c_int * 3)(-1, -1, -1)
        f(L, T, H, HB, group, out)
        assert tuple(out) == items[L]
    assert sorted(items) == sorted((t, h, b) for t in range(T) for h in range(H)
                                   for b in range(B))
    L = 0
    for first in range(0, HB, group):
        pairs = list(range(first, min(first + group, HB)))
        for t in range(T):
            for hb in pairs:
                assert items[L] == (t, hb % H, hb // H), (L, items[L])
                L += 1
    assert L == T * HB


def _packed(shim):
    for f in (shim.shim_packed_grid_tiles, shim.shim_use_packed_grid):
        f.argtypes = [ctypes.c_longlong] * 3
    shim.shim_packed_grid_tiles.restype = ctypes.c_longlong
    shim.shim_use_packed_grid.restype = ctypes.c_int
    return shim.shim_packed_grid_tiles, shim.shim_use_packed_grid


def test_launch_order_beyond_32_bits(shim):
    # a grid of more than 2^32 CTAs takes the 64-bit arithmetic: spot-check the bijection's
    # formula there against the Python model
    T, H, B, group = 2**20, 64, 2**13, 4
    HB = H * B
    for L in (0, 1, 2**32 - 1, 2**32, 2**32 + 12345, T * HB - 1):
        first = L // (group * T) * group
        gn = min(group, HB - first)
        i = L - first * T
        hb = first + i % gn
        assert _grid_item(shim, L, T, H, HB, group) == (i // gn, hb % H, hb // H)


def test_packed_grid_covers_every_tile(shim):
    # The packed varlen grid numbers the 128-row tiles of all segments one after another; its
    # size must cover sum(ceil(L_s / 128)) for every packing of `total` rows into segments
    # no longer than max_len, and never exceed the per-segment grid.
    tiles, _ = _packed(shim)
    rng = np.random.default_rng(5)
    for _ in range(2000):
        nseg = int(rng.integers(1, 300))
        hi = int(rng.choice([1, 60, 128, 129, 700, 5000]))
        lens = rng.integers(0, hi + 1, size=nseg)
        total, mx = int(lens.sum()), int(lens.max())
        need = int(((lens + 127) // 128).sum())
        got = tiles(total, nseg, mx)
        assert need <= got <= nseg * ((mx + 127) // 128), (lens.tolist(), got)
    # tight when every segment is a multiple of 128 rows long and as long as max_len
    assert tiles(64 * 4096, 64, 4096) == 64 * 32


def test_packed_grid_choice(shim):
    _, use = _packed(shim)
    seqlens = wl.varlen_lengths_64(3)
    assert use(sum(seqlens), 64, max(seqlens)) == 1       # the 64-sequence mix: packed
    assert use(64 * 4096, 64, 4096) == 0                   # equal lengths: per segment
    assert use(3 * 1024, 3, 1024) == 0
    assert use(128 + 256 + 512, 3, 512) == 1               # 12 per-segment CTAs for 9 tiles
    assert use(1025 * 10, 1025, 3000) == 0                 # more segments than the scan takes
