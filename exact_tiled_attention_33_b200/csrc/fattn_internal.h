// Internal parameter blocks and launcher declarations shared by the library's
// translation units (not part of the public C ABI in include/fattn.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fattn {

// Forward kernel parameters.  Dense problems have cu_q == nullptr and use B, N;
// varlen problems index sequences through cu_q / cu_k (device int32 prefix sums).
struct FwdParams {
  void* o;          // [B, N, H, D] or [total_q, H, D], 16-bit
  float* lse;       // [B, H, N] or [H, total_q], fp32, natural log
  const int* cu_q;  // varlen only
  const int* cu_k;  // varlen only
  int N;            // dense sequence length
  int H;
  int total_q;      // varlen: rows of q/o (row stride of lse)
  int total_k;      // varlen: rows of k/v
  float scale;      // softmax scale
  float scale_log2; // |scale| * log2(e), > 0 (a tiny positive value when scale == 0)
  int negate_scores;// 1 when scale < 0: the S product negates Q
  float v_descale;  // O is multiplied by it (FP8 inputs; 1 otherwise)
  int win_left;     // attention window (see key_tile_range); causal is (-1, 0)
  int win_right;
  int reverse_tiles;// launch the query tiles with the most key tiles first
  int max_seqlen_q; // varlen: longest allowed segment (longer ones are skipped, reported)
  int num_seqs;     // varlen: segments
  int packed;       // varlen: grid x numbers the tiles of all segments (packed_tile_lookup)
  uint32_t* status; // device status word
};

// Backward kernel parameters (see bwd_kernels.cuh).
struct BwdParams {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;   // as written by the forward pass
  void* dq;
  void* dk;
  void* dv;
  float* dvec;        // D = rowsum(dO ∘ O), same layout as lse (caller's workspace)
  float* dq_acc;      // single-pass backward: fp32 dQ sums (caller's workspace), [rows, H, D]
                      // like dq itself (rows = B*N or total_q)
  const int* cu_q;
  const int* cu_k;
  int B, N, H;
  int total_q, total_k;
  float scale;
  float scale_log2;
  int win_left, win_right;  // attention window (see key_tile_range)
  int reverse_tiles;        // dQ pass: launch the query tiles with the most key tiles first
  int max_seqlen_q, max_seqlen_k;  // varlen: longest allowed segments (longer: skipped, reported)
  int num_seqs;  // varlen: segments
  int packed;    // varlen, single pass: grid x numbers the key tiles of all segments
  uint32_t* status;
};

// Attention window.  Within one sequence of Lq queries and Lk keys (diag = Lk - Lq, the
// bottom-right alignment), key j is allowed for query i iff
//   i + diag - win_left <= j <= i + diag + win_right   and 0 <= j < Lk,
// a negative bound meaning no bound on that side: causal is (-1, 0), full is (-1, -1).
// The callers keep every bound below the sequence lengths and Lq + Lk < 2^31, so none of
// the sums below overflows.

// Key tiles (of BN keys) that query rows [q_first, q_last] may see: tiles
// [*begin, *begin + *count).
__host__ __device__ inline void key_tile_range(int q_first, int q_last, int Lk, int diag,
                                               int win_left, int win_right, int BN, int* begin,
                                               int* count) {
  const int hi = win_right >= 0 ? min(Lk - 1, q_last + diag + win_right) : Lk - 1;
  const int lo = win_left >= 0 ? max(0, q_first + diag - win_left) : 0;
  if (hi < lo) {
    *begin = 0;
    *count = 0;
  } else {
    *begin = lo / BN;
    *count = hi / BN - lo / BN + 1;
  }
}

// Query tiles (of BM rows) that may see keys [k_first, k_last]: tiles
// [*begin, *begin + *count).
__host__ __device__ inline void query_tile_range(int k_first, int k_last, int Lq, int diag,
                                                 int win_left, int win_right, int BM, int* begin,
                                                 int* count) {
  const int lo = win_right >= 0 ? max(0, k_first - diag - win_right) : 0;
  const int hi = win_left >= 0 ? min(Lq - 1, k_last - diag + win_left) : Lq - 1;
  if (hi < lo) {
    *begin = 0;
    *count = 0;
  } else {
    *begin = lo / BM;
    *count = hi / BM - lo / BM + 1;
  }
}

// Work item of the CTA with linear launch index L = x + T (y + H z) on a (T tiles, H heads,
// HB / H batches) grid, in launch order: the (batch, head) pairs are taken `group` at a time,
// and within a group tile-major (tile 0 of each of its heads, then tile 1, ...).  The hardware
// starts CTAs roughly in linear order, so the heads of a group share L2 while they run, and
// the heaviest tiles of the last group start together with the rest of it instead of after
// every other CTA has been handed out.  A bijection of [0, T * HB) onto (tile, h, bz).
struct GridItem {
  int tile, h, bz;
};
// U: the unsigned type the arithmetic runs in (32 bits when the grid fits, which keeps the
// divisions short on the device; 64 bits otherwise).
template <typename U>
__host__ __device__ inline GridItem grouped_grid_item_t(U L, U T, U H, U HB, U group) {
  const U first = L / (group * T) * group;               // first (batch, head) of the group
  const U gn = group < HB - first ? group : HB - first;  // pairs in the group
  const U i = L - first * T;                             // < gn * T
  const U hb = first + i % gn;
  return {(int)(i / gn), (int)(hb % H), (int)(hb / H)};
}
__host__ __device__ inline GridItem grouped_grid_item(unsigned long long L, unsigned long long T,
                                                      unsigned long long H,
                                                      unsigned long long HB,
                                                      unsigned long long group) {
  if (T * HB <= 0xffffffffull && group * T <= 0xffffffffull)
    return grouped_grid_item_t<unsigned>((unsigned)L, (unsigned)T, (unsigned)H, (unsigned)HB,
                                         (unsigned)group);
  return grouped_grid_item_t<unsigned long long>(L, T, H, HB, group);
}

// Packed varlen grid (the device side is packed_tile_lookup): a packing of `total` rows into
// nseg segments has at most (total + 127 nseg) / 128 tiles of 128 rows, and never more than
// the per-segment grid's nseg * ceil(max_len / 128).  The packed grid is used when the
// per-segment grid would launch at least a quarter more CTAs (the surplus ones exit at
// once, after the SM has paid for starting them) and the segments are few enough for the
// per-warp prefix sum.
constexpr long long kPackedMaxSeqs = 1024;
__host__ __device__ inline long long packed_grid_tiles(long long total, long long nseg,
                                                       long long max_len) {
  const long long per_segment = nseg * ((max_len + 127) / 128);
  const long long packed = (total + 127 * nseg) / 128;
  return packed < per_segment ? packed : per_segment;
}
__host__ __device__ inline bool use_packed_grid(long long total, long long nseg,
                                                long long max_len) {
  return nseg <= kPackedMaxSeqs &&
         4 * nseg * ((max_len + 127) / 128) >= 5 * packed_grid_tiles(total, nseg, max_len);
}

#ifdef __CUDACC__
__device__ inline GridItem grouped_tile_order(unsigned group) {
  const unsigned long long T = gridDim.x, H = gridDim.y;
  return grouped_grid_item(blockIdx.x + T * (blockIdx.y + H * blockIdx.z), T, H,
                           H * gridDim.z, group);
}
#endif

// KV-cache decode parameters (see decode_kernel.cuh).
constexpr int kDecodeMaxQueries = 16;  // query rows per sequence in one decode call
struct DecParams {
  const void* q;           // [B, Nq, H, D] 16-bit
  void* o;                 // [B, Nq, H, D] 16-bit
  float* lse;              // [B, H, Nq] fp32, natural log
  const int* seqlens;      // [B] cached rows per sequence (device)
  const int* block_table;  // paged: [B, max_blocks] page ids; contiguous: nullptr
  float* o_part;           // splits > 1: [B, Nq, H, splits, D] fp32 partial outputs
  float* lse_part;         // splits > 1: [B, Nq, H, splits] log2-domain partial LSE
  int B, Nq, H;
  int max_len;             // bound on every seqlens[b] (larger values are clamped, reported)
  int page_size, max_blocks, num_pages;  // paged only
  int splits, chunk;       // CTAs per (sequence, head) and keys per split (multiple of 128)
  float scale_log2;        // scale * log2(e), any sign
  int win_left, win_right; // window as for the forward kernel (causal: -1, 0)
  uint32_t* status;
};

enum class LaunchResult { kOk, kUnsupported, kCudaError };

// The CUDA error behind the calling host thread's last kCudaError (set by the launchers).
cudaError_t& launch_error();

// kOk, or kCudaError with the error recorded for the caller's message.
inline LaunchResult launch_status(cudaError_t e) {
  if (e == cudaSuccess) return LaunchResult::kOk;
  launch_error() = e;
  return LaunchResult::kCudaError;
}

// Forward launch for one problem.  Tensor maps are built by the caller (api.cu).
LaunchResult launch_fwd(int d, bool bf16, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                        const CUtensorMap& tmV, const CUtensorMap& tmO, const FwdParams& p,
                        dim3 grid, cudaStream_t stream);
// FP8 (E4M3) operands, d = 128; bf16 selects the output format.
LaunchResult launch_fwd_fp8(int d, bool bf16, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                            const CUtensorMap& tmV, const CUtensorMap& tmO, const FwdParams& p,
                            dim3 grid, cudaStream_t stream);

// Test-only instance of the forward kernel that writes O in fp32 before rounding (p.o is
// then a float buffer of the same shape).
LaunchResult launch_fwd_f32out(int d, bool bf16, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                               const CUtensorMap& tmV, const CUtensorMap& tmO, const FwdParams& p,
                               dim3 grid, cudaStream_t stream);

// Query rows per forward CTA (grid x = ceil(rows / this), y = heads, z = batch or
// sequences): one 128-row tile.
int fwd_rows_per_cta(bool fp8);

// Decode launch: the split kernel and, when p.splits > 1, the merge kernel.
LaunchResult launch_decode(int d, bool bf16, bool paged, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const DecParams& p, cudaStream_t stream);

// Tensor maps of the single-pass backward: q, k, v, dout as for launch_bwd; dq over the
// fp32 dQ sums p.dq_acc ([rows, H, D]; box 32 columns x 1 head x 128 rows, 128-byte
// swizzle) that the pass reduce-adds its dQ partials through; dk, dv over the 16-bit
// gradients (layout and box of k, v) that whole key tiles are stored through.
struct BwdFusedMaps {
  CUtensorMap q, k, v, dout, dq, dk, dv;
};

// Single-pass backward launch: D preprocess (and zeroing of the dQ sums), the fused
// dK/dV/dQ pass, the dQ conversion.  q_rows and batches as for launch_bwd.
LaunchResult launch_bwd_fused(int d, bool bf16, const BwdFusedMaps& m, const BwdParams& p,
                              long long q_rows, int max_seqlen_k, int batches,
                              cudaStream_t stream);

// Backward launch: D preprocess, dK/dV pass, dQ pass.  q_rows = B*N (dense) or total_q
// (varlen); batches = B (dense) or num_seqs (varlen).
LaunchResult launch_bwd(int d, bool bf16, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                        const CUtensorMap& tmV, const CUtensorMap& tmDO, const BwdParams& p,
                        long long q_rows, int max_seqlen_q, int max_seqlen_k, int batches,
                        cudaStream_t stream);

}  // namespace fattn
