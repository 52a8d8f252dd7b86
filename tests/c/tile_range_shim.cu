// Host-callable wrappers of the kernels' tile-range helpers, so that the CPU tests can
// check which K/V (or Q) tiles a tile visits against the oracle's attention mask.
#include "fattn_internal.h"

extern "C" void shim_key_tile_range(int q_first, int q_last, int Lk, int diag, int win_left,
                                    int win_right, int BN, int* begin, int* count) {
  fattn::key_tile_range(q_first, q_last, Lk, diag, win_left, win_right, BN, begin, count);
}

extern "C" void shim_query_tile_range(int k_first, int k_last, int Lq, int diag, int win_left,
                                      int win_right, int BM, int* begin, int* count) {
  fattn::query_tile_range(k_first, k_last, Lq, diag, win_left, win_right, BM, begin, count);
}

