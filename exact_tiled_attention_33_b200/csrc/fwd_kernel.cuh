// Forward pass of exact attention, tile by tile with online softmax, for sm_100a.
//
// Method (what is computed): the tiled algorithm of the page
// "FlashAttention实战：如何在A100上实现3倍加速的Transformer训练" §2 and §3 — an outer loop
// over query tiles, an inner loop over key/value tiles, and per query row a running
// maximum m and a running sum l that are rescaled as each new tile arrives (§3.1),
// fused with both matrix products so that scores never leave the chip (§3.2).  The
// output accumulator is rescaled by the same factor as l; it is divided by l once at
// the end, and the row's log-sum-exp is stored for the backward pass (page
// "Flash Attention V3：大模型训练加速与显存优化技术解析" §3.2: O(N) saved state).
//
// How it maps to B200 (the pages' A100/H100 block sizes are not used):
//   * one CTA owns one query tile of BM = 128 rows and walks the key/value tiles
//     (BN = 128 keys) its rows may see;
//   * warp 0 issues TMA loads (Q once; K and V through a STAGES-deep ring);
//   * warp 1, one thread, issues tcgen05.mma: S_j = Q K_jᵀ into one of two tensor-memory
//     buffers (so S_{j+1} is computed while the softmax of S_j runs), and O += P_j V_j
//     with P_j read from tensor memory;
//   * warps 4..7 and 8..11 are two softmax warpgroups working on the same tile: thread r
//     of each owns row r (= tensor-memory lane r) and one half (64) of its 128 scores.
//     The halves combine their row maxima through shared memory (one named barrier per
//     tile), update the reference maximum m identically, and keep partial row sums;
//     each writes P over its own S columns as packed 16-bit values and rescales its half
//     of O only when m grew by more than 2^8 (exact: O and l share the reference);
//   * tensor memory: S_a | S_b | O (128 + 128 + D + 16 columns of 32 bits); the P·V
//     product runs with 16 more columns of V that are all ones, so O's last 16 columns
//     hold the row sum of the rounded P it used (the normaliser of O);
//   * FP8 = true: E4M3 operands and 8-bit tensor-core products (d = 128).
#pragma once

#include <type_traits>

#include "fattn_internal.h"
#include "sm100.cuh"

namespace fattn {

// FP8: E4M3 operands (1 byte) and 8-bit MMAs (32 elements of K per instruction).
template <int D, bool FP8 = false>
struct FwdCfg {
  static constexpr int BM = 128;  // query rows per tile = tensor-memory lanes
  static constexpr int BN = 128;  // keys per K/V tile
  static constexpr int EB = FP8 ? 1 : 2;        // operand bytes
  static constexpr int KSTEP = FP8 ? 32 : 16;   // K elements per MMA instruction
  static constexpr int STAGES = FP8 ? 4 : ((D == 128) ? 2 : 4);
  static constexpr int KCH = D * EB / 128;      // 128-byte column chunks per row
  static constexpr int CHUNK = 128 * 128;
  static constexpr int TILE = 128 * D * EB;
  // Each V stage carries one more 128-byte column chunk filled with ones: the P·V product
  // then also yields, in O columns D..D+15, the row sum of the rounded P it used.
  static constexpr int NO = D + 16;                    // O columns in tensor memory
  static constexpr int VSTAGE = (KCH + 1) * CHUNK;     // V tile + the ones chunk
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE;
  static constexpr int OFF_V = OFF_K + STAGES * TILE;
  static constexpr int OFF_RED = OFF_V + STAGES * VSTAGE;  // max exchange [2][2][128], sums [2][128]
  static constexpr int OFF_BAR = OFF_RED + 4 * 2 * 128 * 4;
  static constexpr int B_QFULL = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_KEMPTY = B_KFULL + STAGES;
  static constexpr int B_VFULL = B_KEMPTY + STAGES;
  static constexpr int B_VEMPTY = B_VFULL + STAGES;
  static constexpr int B_SFULL = B_VEMPTY + STAGES;
  static constexpr int B_PFULL = B_SFULL + 2;
  static constexpr int B_ODONE = B_PFULL + 1;
  static constexpr int NBAR = B_ODONE + 1;
  static constexpr int SMEM_BYTES = OFF_BAR + 8 * NBAR + 16 + 1024;  // + alignment slack
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static constexpr int THREADS = 384;  // warps 0 loads, 1 MMA, 2-3 idle, 4-11 softmax
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_O = 256;
  // pairs of every 16 (per 32-column chunk) whose exponentials use exp2_poly2.  At d = 64
  // a score carries half the tensor work of d = 128 for the same exponential, so a larger
  // share moves to the FMA pipe there.
#ifndef FATTN_POLY_PAIRS
#define FATTN_POLY_PAIRS 4
#endif
#ifndef FATTN_POLY_PAIRS_D64
#define FATTN_POLY_PAIRS_D64 6
#endif
  static constexpr int kPolyPairs = D == 64 ? FATTN_POLY_PAIRS_D64 : FATTN_POLY_PAIRS;
  // packed P column for the kk-th K step of a 128-key tile.  16-bit P (16 keys per step,
  // 2 per column): half 0 packs into columns 0..31 of its S buffer, half 1 into 64..95.
  // 8-bit P (32 keys per step, 4 per column): half 0 into 0..15, half 1 into 64..79.
  __device__ static constexpr uint32_t packed_col(int kk) {
    return FP8 ? (uint32_t)((kk >> 1) * 64 + (kk & 1) * 8)
               : (uint32_t)(kk * 8 + (kk >= 4 ? 32 : 0));
  }
};

// BF16: 16-bit format of the output (and of the operands unless FP8).  F32O: the output is
// written in fp32 before any rounding (a test-only instance: the library's entry points
// all write 16-bit O; fa_selftest_fwd_f32 exposes this one to the parity tests).
// The check of every segment that the packed grid's first CTA makes, kept out of line: inlined
// into the kernel body it slowed the main loop of the instance that contains it by about 10%.
static __device__ __noinline__ void varlen_check_all_out_of_line(const int* cu_q,
                                                                 const int* cu_k, int nseg,
                                                                 int total_q, int total_k,
                                                                 long long q_cover,
                                                                 uint32_t* status) {
  varlen_check_all(cu_q, cu_k, nseg, total_q, total_k, q_cover, -1, status);
}

// PACKED: the packed varlen grid (packed_tile_lookup).  A separate instance, because the
// lookup's code in the kernel body slowed the main loop of every launch by about 10%.
template <int D, bool BF16, bool FP8 = false, bool F32O = false, bool PACKED = false>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams p) {
  using C = FwdCfg<D, FP8>;
  constexpr int EL = 128 / C::EB;  // elements per 128-byte chunk (TMA x step)
  // 8-bit P is scaled by 2^6 (p = 2^(x - m + 6)) so that it spans the normal E4M3 range,
  // and the reference maximum is refreshed once the row maximum grows by more than 2.5, so
  // that p stays below 2^8.5 < 448; 16-bit P keeps p = 2^(x - m) with the lazy threshold 8.
  constexpr float POFF = FP8 ? 6.f : 0.f;
  constexpr float LAZY = FP8 ? 2.5f : 8.f;
  constexpr int BM = C::BM, BN = C::BN, ST = C::STAGES;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + C::OFF_BAR + 8 * C::NBAR);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  float* red = reinterpret_cast<float*>(sgen + C::OFF_RED);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---------------------------------------------------------------- work item
  // grid: x = query tile, y = head, z = batch or sequence (a packed varlen grid: x = the
  // query tiles of all sequences, z = 1), launched in groups of heads that share L2 (see
  // grouped_tile_order); when causal the tile with the most key tiles of each head (or of
  // each sequence) comes first.
#ifndef FATTN_FWD_HEAD_GROUP
#define FATTN_FWD_HEAD_GROUP 4
#endif
  const GridItem item = grouped_tile_order(FATTN_FWD_HEAD_GROUP);
  const int h = item.h;
  int bz = item.bz;
  int tile = p.reverse_tiles ? (int)(gridDim.x - 1) - item.tile : item.tile;
  int Lq, Lk, q_row0, k_row0, bcoord;
  if (p.cu_q != nullptr) {
    if constexpr (PACKED) {  // x numbers the query tiles of all segments, one after another
      if (blockIdx.x == 0 && blockIdx.y == 0)
        varlen_check_all_out_of_line(p.cu_q, p.cu_k, p.num_seqs, p.total_q, p.total_k,
                                     p.max_seqlen_q, p.status);
      if (!packed_tile_lookup(p.cu_q, p.num_seqs, p.total_q, item.tile, &bz, &tile)) return;
    }
    if (!varlen_segment_ok(p.cu_q, p.cu_k, bz, p.total_q, p.total_k, p.max_seqlen_q, -1,
                           p.status))
      return;
    q_row0 = p.cu_q[bz];
    Lq = p.cu_q[bz + 1] - q_row0;
    if constexpr (PACKED)
      if (p.reverse_tiles) tile = (Lq + BM - 1) / BM - 1 - tile;
    k_row0 = p.cu_k[bz];
    Lk = p.cu_k[bz + 1] - k_row0;
    bcoord = 0;
  } else {
    q_row0 = 0;
    k_row0 = 0;
    Lq = Lk = p.N;
    bcoord = bz;
  }
  const int q0 = tile * BM;
  if (q0 >= Lq) return;  // uniform for the whole CTA
  const int diag = Lk - Lq;  // bottom-right alignment of the window (causal: j <= i + diag)
  const int wl = p.win_left, wr = p.win_right;
  int j0, n_kv;               // key tiles j0 .. j0 + n_kv - 1
  key_tile_range(q0, min(q0 + BM - 1, Lq - 1), Lk, diag, wl, wr, BN, &j0, &n_kv);

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_QFULL), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(BAR(C::B_KFULL + s), 1);
      mbar_init(BAR(C::B_KEMPTY + s), 1);
      mbar_init(BAR(C::B_VFULL + s), 1);
      mbar_init(BAR(C::B_VEMPTY + s), 1);
    }
    mbar_init(BAR(C::B_SFULL), 1);
    mbar_init(BAR(C::B_SFULL + 1), 1);
    mbar_init(BAR(C::B_PFULL), 256);
    mbar_init(BAR(C::B_ODONE), 1);
    *abort_flag = 0u;
    fence_barrier_init();
    // Thread 0 is the TMA producer's lane: Q and the first K/V stages are requested right
    // away, so their DRAM latency overlaps the tensor-memory allocation and the setup
    // barrier (fresh stages need no EMPTY wait; the ones chunk written below lies outside
    // the V tile's chunks).
    if (n_kv > 0) {
      mbar_arrive_expect_tx(BAR(C::B_QFULL), C::TILE);
      for (int c = 0; c < C::KCH; ++c)
        tma_load_4d(&tmQ, BAR(C::B_QFULL), sbase + C::OFF_Q + c * C::CHUNK, c * EL, h, q_row0 + q0,
                    bcoord);
      for (int j = 0; j < min(ST, n_kv); ++j) {
        mbar_arrive_expect_tx(BAR(C::B_KFULL + j), C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(&tmK, BAR(C::B_KFULL + j), sbase + C::OFF_K + j * C::TILE + c * C::CHUNK,
                      c * EL, h, k_row0 + (j0 + j) * BN, bcoord);
        mbar_arrive_expect_tx(BAR(C::B_VFULL + j), C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(&tmV, BAR(C::B_VFULL + j), sbase + C::OFF_V + j * C::VSTAGE + c * C::CHUNK,
                      c * EL, h, k_row0 + (j0 + j) * BN, bcoord);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  {
    // the ones chunk of every V stage (1.0 in the operand format), for the tensor core
    const uint32_t one = FP8 ? 0x38383838u : (BF16 ? 0x3F803F80u : 0x3C003C00u);
    for (int e = threadIdx.x; e < ST * (C::CHUNK / 16); e += C::THREADS) {
      const int s = e / (C::CHUNK / 16), w = e % (C::CHUNK / 16);
      *reinterpret_cast<uint4*>(sgen + C::OFF_V + s * C::VSTAGE + C::KCH * C::CHUNK + w * 16) =
          make_uint4(one, one, one, one);
    }
    fence_proxy_async_smem();  // visible to the tensor core (async proxy)
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0 && n_kv > 0) {
      // Q and key tiles 0 .. ST-1 were requested during setup
      for (int j = ST; j < n_kv; ++j) {
        const int s = j % ST;
        const uint32_t ph = (uint32_t)(j / ST) & 1u;
        mbar_wait(BAR(C::B_KEMPTY + s), ph ^ 1u, abort_flag, p.status);
        mbar_arrive_expect_tx(BAR(C::B_KFULL + s), C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(&tmK, BAR(C::B_KFULL + s), sbase + C::OFF_K + s * C::TILE + c * C::CHUNK,
                      c * EL, h, k_row0 + (j0 + j) * BN, bcoord);
        mbar_wait(BAR(C::B_VEMPTY + s), ph ^ 1u, abort_flag, p.status);
        mbar_arrive_expect_tx(BAR(C::B_VFULL + s), C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(&tmV, BAR(C::B_VFULL + s), sbase + C::OFF_V + s * C::VSTAGE + c * C::CHUNK,
                      c * EL, h, k_row0 + (j0 + j) * BN, bcoord);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0 && n_kv > 0) {
      // S = Q Kᵀ: A = Q (K-major), B = K (K-major).  O += P V: A = P (tensor memory),
      // B = V stored [key][d], i.e. N-contiguous (MN-major).
      // (format code 0 is f16 for .kind::f16 and E4M3 for .kind::f8f6f4)
      constexpr uint32_t ID_S0 = idesc_f16_f32acc(BF16 && !FP8, BM, BN, false, false);
      const uint32_t ID_S = ID_S0 | (p.negate_scores ? (1u << 13) : 0u);  // bit 13: negate A
      constexpr uint32_t ID_O = idesc_f16_f32acc(BF16 && !FP8, BM, C::NO, false, true);
      // Descriptors built once; each MMA only adds a compile-time offset.
      const uint64_t dQ = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);
      const uint64_t dK0 = sdesc_sw128(sbase + C::OFF_K, 16, 1024);
      const uint64_t dV0 = sdesc_sw128(sbase + C::OFF_V, C::CHUNK, 1024);
      auto issue_s = [&](int j) {  // S_j into buffer j % 2
        const int s = j % ST;
        mbar_wait(BAR(C::B_KFULL + s), (uint32_t)(j / ST) & 1u, abort_flag, p.status);
        tc_fence_after();
        const uint64_t db = sdesc_adv(dK0, (uint32_t)(s * C::TILE));
        const uint32_t dst = tmem + 128u * (uint32_t)(j & 1);
#pragma unroll
        for (int kk = 0; kk < D / C::KSTEP; ++kk) {
          // K step kk starts kk * 32 bytes into the rows: chunk kk / 4, byte (kk % 4) * 32
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          if constexpr (FP8)
            mma_ss_f8(dst, sdesc_adv(dQ, off), sdesc_adv(db, off), ID_S, kk > 0 ? 1u : 0u);
          else
            mma_ss(dst, sdesc_adv(dQ, off), sdesc_adv(db, off), ID_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(BAR(C::B_SFULL + (j & 1)));
        mma_commit(BAR(C::B_KEMPTY + s));
      };
      mbar_wait(BAR(C::B_QFULL), 0, abort_flag, p.status);
      issue_s(0);
      if (n_kv > 1) issue_s(1);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % ST;
        mbar_wait(BAR(C::B_PFULL), (uint32_t)j & 1u, abort_flag, p.status);
        mbar_wait(BAR(C::B_VFULL + s), (uint32_t)(j / ST) & 1u, abort_flag, p.status);
        tc_fence_after();
        const uint64_t db = sdesc_adv(dV0, (uint32_t)(s * C::VSTAGE));
        const uint32_t src = tmem + 128u * (uint32_t)(j & 1);
#pragma unroll
        for (int kk = 0; kk < BN / C::KSTEP; ++kk) {
          // V rows kk * KSTEP .. of the tile: 128-byte rows, so KSTEP * 128 bytes per step
          if constexpr (FP8)
            mma_ts_f8(tmem + C::TM_O, src + C::packed_col(kk),
                      sdesc_adv(db, kk * C::KSTEP * 128), ID_O, (j > 0 || kk > 0) ? 1u : 0u);
          else
            mma_ts(tmem + C::TM_O, src + C::packed_col(kk), sdesc_adv(db, kk * C::KSTEP * 128),
                   ID_O, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(BAR(C::B_ODONE));
        mma_commit(BAR(C::B_VEMPTY + s));
        // S_{j+2} reuses the buffer of S_j, whose P the product above has just consumed
        // (tcgen05.mma from one thread run in order).
        if (j + 2 < n_kv) issue_s(j + 2);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ============================================================ softmax warpgroups
    const int half = (warp - 4) >> 2;  // score columns 64*half .. 64*half+63
    const int quarter = warp & 3;      // tensor-memory lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int i = q0 + row;            // this thread's query row
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float c = p.scale_log2;      // > 0: scores are handled as x = s * |scale| * log2(e)
    float m = -INFINITY;               // reference maximum of x shared by l and O
    float l = 0.f;                     // Σ p over this half's columns (fp32), for the LSE
    // (the row sum of the rounded P that normalises O accumulates in O's extra columns)
    float* red_max = red;              // [parity][half][row]
    float* red_sum = red + 2 * 2 * 128;  // [half][row]: l at the end

    for (int j = 0; j < n_kv; ++j) {
      const int b = j & 1;
      mbar_wait(BAR(C::B_SFULL + b), (uint32_t)(j >> 1) & 1u, abort_flag, p.status);
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + 128u * (uint32_t)b + 64u * (uint32_t)half;
      uint32_t sr[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      reg_fence(sr);

      const int kt = (j0 + j) * BN;       // first key of the tile
      const int k0 = kt + 64 * half;      // first key of this thread's columns
      const bool need_mask = (kt + BN > Lk) || (wr >= 0 && kt + BN - 1 > q0 + diag + wr) ||
                             (wl >= 0 && kt < q0 + BM - 1 + diag - wl);
      if (need_mask) {
        // allowed columns: lo <= e < lim
        const int lim = wr >= 0 ? min(Lk - k0, i + diag + wr - k0 + 1) : Lk - k0;
        const int lo = wl >= 0 ? i + diag - wl - k0 : 0;
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (e >= lim || e < lo) sr[e] = __float_as_uint(-INFINITY);
      }
      // partial row maximum (tree of 3-input maxima), combined with the other half's
      float t1[22];
#pragma unroll
      for (int e = 0; e < 21; ++e)
        t1[e] = fmax3(__uint_as_float(sr[3 * e]), __uint_as_float(sr[3 * e + 1]),
                      __uint_as_float(sr[3 * e + 2]));
      t1[21] = __uint_as_float(sr[63]);
      float t2[8];
#pragma unroll
      for (int e = 0; e < 7; ++e) t2[e] = fmax3(t1[3 * e], t1[3 * e + 1], t1[3 * e + 2]);
      t2[7] = t1[21];
      const float pm = fmax3(fmax3(t2[0], t2[1], t2[2]), fmax3(t2[3], t2[4], t2[5]),
                             fmaxf(t2[6], t2[7]));
      red_max[(b * 2 + half) * 128 + row] = pm;
      named_barrier_sync(1, 256);
      const float mx = fmaxf(pm, red_max[(b * 2 + (half ^ 1)) * 128 + row]) * c;

      // Reference-maximum update (identical in both halves).  Keep the stale maximum
      // while the new one exceeds it by at most 8 (a factor 2^8 in P, harmless in fp32).
      bool rescale = false;
      float alpha = 1.f;
      if (m == -INFINITY) {
        m = mx;  // first allowed keys for this row: O and l are still exactly 0
      } else if (mx - m > LAZY) {
        alpha = ex2_approx(m - mx);
        m = mx;
        rescale = true;
      }
      const float m_use = (m == -INFINITY) ? 0.f : m;
      // p = 2^(s*c - m).  l sums the fp32 p (log-sum-exp).  O is normalised by the row sum
      // of the rounded P that the P·V product itself accumulates in O's extra columns, so
      // numerator and denominator share the rounding of P (under the lazy maximum the
      // largest P of a row is 2^δ, not 1).
      const uint64_t c2 = f2_pack(c, c);
      const uint64_t nm2 = f2_pack(POFF - m_use, POFF - m_use);
      uint64_t ls2 = 0ull;
      // kPolyPairs of every 16 pairs of exponentials run on the FMA pipe (tiles without
      // masked keys), the rest on the special-function unit; the choice is made once per
      // tile so the loop bodies stay branch-free.
      auto exp_pass = [&](auto use_poly) {
        [[maybe_unused]] uint32_t pk8[16];  // 8-bit P: four keys per 32-bit column
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          [[maybe_unused]] uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sr[q * 32 + 2 * e]),
                                               __uint_as_float(sr[q * 32 + 2 * e + 1])),
                                       c2, nm2);
            const float2 xx = f2_unpack(x2);
            float p0, p1;
            if (decltype(use_poly)::value && e < C::kPolyPairs) {
              const float2 pp = exp2_poly2(xx.x, xx.y);
              p0 = pp.x;
              p1 = pp.y;
            } else {
              p0 = ex2_approx(xx.x);
              p1 = ex2_approx(xx.y);
            }
            if constexpr (FP8) {
              const uint32_t h8 = pack2_e4m3(p0, p1);
              if (e & 1)
                pk8[q * 8 + (e >> 1)] |= h8 << 16;
              else
                pk8[q * 8 + (e >> 1)] = h8;
            } else {
              pk[e] = pack2<BF16>(p0, p1);
            }
            ls2 = f2_add(ls2, f2_pack(p0, p1));
          }
          if constexpr (!FP8) tmem_st16(tS + q * 16, pk);
        }
        if constexpr (FP8) tmem_st16(tS, pk8);
      };
      if (need_mask)
        exp_pass(std::false_type{});
      else
        exp_pass(std::true_type{});
      const float2 ls = f2_unpack(ls2);
      l = l * alpha + (ls.x + ls.y);

      if (__any_sync(0xffffffffu, rescale)) {
        // O was last written by the P·V product of tile j-1: wait until it completed, then
        // rescale this half's columns of O.
        mbar_wait(BAR(C::B_ODONE), (uint32_t)(j - 1) & 1u, abort_flag, p.status);
        tc_fence_after();
        const uint32_t tO = tmem + lane_off + C::TM_O + (uint32_t)(half * (D / 2));
#pragma unroll 1
        for (int q = 0; q < D / 64; ++q) {
          uint32_t o[32];
          tmem_ld32(tO + q * 32, o);
          tmem_wait_ld();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + q * 32, o);
        }
        if (half == 1) {  // the rounded-P row sum columns D..D+15 scale with O
          uint32_t o[16];
          tmem_ld16(tmem + lane_off + C::TM_O + D, o);
          tmem_wait_ld();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st16(tmem + lane_off + C::TM_O + D, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(C::B_PFULL));
    }

    // ---------------------------------------------------------------- epilogue
    if (n_kv > 0) {
      mbar_wait(BAR(C::B_ODONE), (uint32_t)(n_kv - 1) & 1u, abort_flag, p.status);
      tc_fence_after();
    }
    red_sum[half * 128 + row] = l;
    named_barrier_sync(1, 256);
    const float L = l + red_sum[(half ^ 1) * 128 + row];
    float LR = 0.f;  // row sum of the rounded P (O column D)
    if (n_kv > 0) {
      uint32_t o[16];
      tmem_ld16(tmem + lane_off + C::TM_O + D, o);
      tmem_wait_ld();
      reg_fence(o);
      LR = __uint_as_float(o[0]);
    }
    const bool valid = i < Lq;
    const float inv_l = (LR > 0.f) ? p.v_descale / LR : 0.f;
    const size_t orow_idx = (p.cu_q != nullptr) ? ((size_t)(q_row0 + i) * p.H + h) * D
                                                : (((size_t)bcoord * p.N + i) * p.H + h) * D;
    uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) + orow_idx;
    // Whole query tiles (and every dense tile: rows past N lie outside the tensor map) leave
    // through shared memory: each thread writes its row into the K stages, free once the
    // last P·V product completed (every S product before it has), in the 128-byte swizzled
    // layout, and one TMA store per 64-column chunk writes whole rows.  The last, partial
    // tile of a packed sequence is stored row by row instead, so that it leaves the next
    // sequence's rows alone.
    const bool via_tma = !F32O && (p.cu_q == nullptr || q0 + BM <= Lq);
    // this half stores O columns [half * D/2, (half + 1) * D/2)
#pragma unroll 1
    for (int q = half * (D / 64); q < (half + 1) * (D / 64); ++q) {
      uint32_t o[32];
      if (n_kv > 0) {
        tmem_ld32(tmem + lane_off + C::TM_O + q * 32, o);
        tmem_wait_ld();
        reg_fence(o);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if constexpr (F32O) {
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.o) + orow_idx + q * 32);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            dst[v4] = make_float4(__uint_as_float(o[4 * v4]) * inv_l, __uint_as_float(o[4 * v4 + 1]) * inv_l,
                                  __uint_as_float(o[4 * v4 + 2]) * inv_l, __uint_as_float(o[4 * v4 + 3]) * inv_l);
        }
        continue;
      }
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pk[e] = pack2<BF16>(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
      if (via_tma) {
        // 16-byte unit u of row r of a chunk sits at r * 128 + ((u ^ (r % 8)) * 16)
        uint8_t* srow = sgen + C::OFF_K + (q >> 1) * C::CHUNK + row * 128;
        const int u0 = (q & 1) * 4;
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          *reinterpret_cast<uint4*>(srow + (((u0 + v4) ^ (row & 7)) << 4)) =
              make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
      } else if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
      }
    }
    if (via_tma) {  // uniform over the CTA
      fence_proxy_async_smem();  // the rows above, visible to the TMA unit
      named_barrier_sync(1, 256);
      if (warp == 4 && lane == 0) {
        for (int c = 0; c < D / 64; ++c)
          tma_store_4d(&tmO, sbase + C::OFF_K + c * C::CHUNK, c * 64, h, q_row0 + q0, bcoord);
        bulk_commit_group();
        bulk_wait_group_read0();  // shared memory stays allocated until the TMA has read it
      }
    }
    if (valid && half == 0) {
      const float lse =
          (L > 0.f) ? (m - POFF + lg2_approx(L)) * 0.69314718055994530942f : INFINITY;
      if (p.cu_q != nullptr)
        p.lse[(size_t)h * p.total_q + q_row0 + i] = lse;
      else
        p.lse[((size_t)bcoord * p.H + h) * p.N + i] = lse;
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fattn
