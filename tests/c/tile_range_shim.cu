// Host-callable wrappers of the kernels' tile-range helpers, so that the CPU tests can
// check which K/V (or Q) tiles a tile visits against the oracle's attention mask, and of the
// launch-order map from a CTA's linear index to its (tile, head, batch), and of the packed
// varlen grid's size rule.
#include "fattn_internal.h"

extern "C" void shim_key_tile_range(int q_first, int q_last, int Lk, int diag, int win_left,
                                    int win_right, int BN, int* begin, int* count) {
  fattn::key_tile_range(q_first, q_last, Lk, diag, win_left, win_right, BN, begin, count);
}

extern "C" void shim_query_tile_range(int k_first, int k_last, int Lq, int diag, int win_left,
                                      int win_right, int BM, int* begin, int* count) {
  fattn::query_tile_range(k_first, k_last, Lq, diag, win_left, win_right, BM, begin, count);
}

extern "C" void shim_grouped_grid_item(unsigned long long L, unsigned long long T,
                                       unsigned long long H, unsigned long long HB,
                                       unsigned long long group, int* out3) {
  const fattn::GridItem g = fattn::grouped_grid_item(L, T, H, HB, group);
  out3[0] = g.tile;
  out3[1] = g.h;
  out3[2] = g.bz;
}

extern "C" long long shim_packed_grid_tiles(long long total, long long nseg, long long max_len) {
  return fattn::packed_grid_tiles(total, nseg, max_len);
}

extern "C" int shim_use_packed_grid(long long total, long long nseg, long long max_len) {
  return fattn::use_packed_grid(total, nseg, max_len) ? 1 : 0;
}

extern "C" void shim_grouped_grid_item_u64(unsigned long long L, unsigned long long T,
                                           unsigned long long H, unsigned long long HB,
                                           unsigned long long group, int* out3) {
  const fattn::GridItem g =
      fattn::grouped_grid_item_t<unsigned long long>(L, T, H, HB, group);
  out3[0] = g.tile;
  out3[1] = g.h;
  out3[2] = g.bz;
}
