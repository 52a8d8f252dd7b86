// Forward pass of exact attention for sm_100a with two query tiles per CTA.
//
// What is computed is the same as fa_fwd_kernel (fwd_kernel.cuh): the tiled online softmax
// of page "FlashAttention实战：如何在A100上实现3倍加速的Transformer训练" §3 — a running row
// maximum and a rescaled running sum per query row, both products fused with the softmax —
// and the row's log-sum-exp for the backward pass (page "Flash Attention V3：大模型训练加速与
// 显存优化技术解析" §3.2).
//
// How it maps to B200:
//   * one CTA owns two 128-row query tiles (rows q0 .. q0 + 255) and walks the union of the
//     128-key tiles they may see; each K/V tile read from shared memory serves both;
//   * warp 0 issues TMA loads (Q0 and Q1 once; K through a KST-deep ring, V VST-deep);
//   * warp 1, one thread, issues every tcgen05.mma, alternating between the tiles:
//     S0 = Q0 Kᵀ, S1 = Q1 Kᵀ, then per key tile O0 += P0 V, S0' = Q0 K'ᵀ, O1 += P1 V,
//     S1' = Q1 K'ᵀ, so the tensor core works on one tile while the other tile's softmax runs;
//   * warps 4..7 are the softmax warpgroup of tile 0, warps 8..11 that of tile 1: thread r
//     owns row r (= tensor-memory lane r) and all 128 scores of a key tile, so no row
//     statistic is exchanged between warps.  A row's scores are read from tensor memory
//     three times per key tile: all 128 at once for the row maximum, then 64 at a time for
//     the exponentials (all 128 plus the exponentials' temporaries exceed the 168 registers
//     a thread has with 12 warps);  P is written over its own S columns as packed
//     16-bit values and read by the P·V product from tensor memory.  The reference maximum m
//     is refreshed only when the row maximum grows by more than 2^8 (O and l share it, so
//     this is exact); O is then rescaled in tensor memory.  The row sum that normalises O is
//     taken over the rounded 16-bit P the product used, the LSE's over the fp32 p;
//   * tensor memory: S0 | S1 | O0 | O1 (128 + 128 + D + D columns).
#pragma once

#include <type_traits>

#include "fattn_internal.h"
#include "sm100.cuh"

namespace fattn {

template <int D>
struct Fwd2Cfg {
  static constexpr int BM = 128;  // query rows per tile (two tiles per CTA)
  static constexpr int BN = 128;  // keys per K/V tile
  static constexpr int KST = D == 128 ? 3 : 4;  // K ring stages
  static constexpr int VST = D == 128 ? 2 : 4;  // V ring stages
  static constexpr int KCH = D / 64;            // 128-byte column chunks per row
  static constexpr int CHUNK = 128 * 128;
  static constexpr int TILE = 128 * D * 2;
  static constexpr int OFF_Q = 0;                      // Q0, Q1
  static constexpr int OFF_K = OFF_Q + 2 * TILE;
  static constexpr int OFF_V = OFF_K + KST * TILE;
  static constexpr int OFF_BAR = OFF_V + VST * TILE;
  static constexpr int B_QFULL = 0;                    // 2
  static constexpr int B_KFULL = 2;
  static constexpr int B_KEMPTY = B_KFULL + KST;
  static constexpr int B_VFULL = B_KEMPTY + KST;
  static constexpr int B_VEMPTY = B_VFULL + VST;
  static constexpr int B_SFULL = B_VEMPTY + VST;       // 2
  static constexpr int B_PFULL = B_SFULL + 2;          // 2
  static constexpr int B_ODONE = B_PFULL + 2;          // 2
  static constexpr int NBAR = B_ODONE + 2;
  static constexpr int SMEM_BYTES = OFF_BAR + 8 * NBAR + 16 + 1024;  // + alignment slack
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static constexpr int THREADS = 384;  // warps 0 loads, 1 MMA, 2-3 idle, 4-7 / 8-11 softmax
  static constexpr int W_LOAD = 0, W_MMA = 1;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_S = 0;    // + 128 * tile
  static constexpr uint32_t TM_O = 256;  // + D * tile
#ifndef FATTN_POLY_PAIRS
#define FATTN_POLY_PAIRS 2
#endif
#ifndef FATTN_POLY_PAIRS_D64
#define FATTN_POLY_PAIRS_D64 6
#endif
  // pairs of every 16 whose exponentials run on the FMA pipe (exp2_poly2)
  static constexpr int kPolyPairs = D == 64 ? FATTN_POLY_PAIRS_D64 : FATTN_POLY_PAIRS;
};

// F32O: O written in fp32 before rounding (test-only instance, fa_selftest_fwd_f32).
template <int D, bool BF16, bool F32O = false>
__global__ void __launch_bounds__(384, 1)
    fa_fwd2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = Fwd2Cfg<D>;
  constexpr int BM = C::BM, BN = C::BN, KST = C::KST, VST = C::VST;
  constexpr float LAZY = 8.f;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + C::OFF_BAR + 8 * C::NBAR);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---------------------------------------------------------------- work item
  // grid: x = pair of query tiles (fastest, so CTAs running together share one head's K/V
  // in L2), y = head, z = batch or sequence; causal-style windows launch the pair with the
  // most key tiles first.
  const int h = blockIdx.y;
  const int bz = blockIdx.z;
  const int pair = p.reverse_tiles ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
  int Lq, Lk, q_row0, k_row0, bcoord;
  if (p.cu_q != nullptr) {
    if (!varlen_segment_ok(p.cu_q, p.cu_k, bz, p.total_q, p.total_k, p.max_seqlen_q, -1,
                           p.status))
      return;
    q_row0 = p.cu_q[bz];
    Lq = p.cu_q[bz + 1] - q_row0;
    k_row0 = p.cu_k[bz];
    Lk = p.cu_k[bz + 1] - k_row0;
    bcoord = 0;
  } else {
    q_row0 = 0;
    k_row0 = 0;
    Lq = Lk = p.N;
    bcoord = bz;
  }
  const int qp = pair * 2 * BM;  // first row of tile 0
  if (qp >= Lq) return;          // uniform for the whole CTA
  const int diag = Lk - Lq;
  const int wl = p.win_left, wr = p.win_right;
  // key tiles of each query tile: [ja[t], ja[t] + na[t]); tile 1 may be empty
  int ja[2], na[2];
  key_tile_range(qp, min(qp + BM - 1, Lq - 1), Lk, diag, wl, wr, BN, &ja[0], &na[0]);
  if (qp + BM < Lq) {
    key_tile_range(qp + BM, min(qp + 2 * BM - 1, Lq - 1), Lk, diag, wl, wr, BN, &ja[1], &na[1]);
  } else {
    ja[1] = 0;
    na[1] = 0;
  }
  // union of the two ranges (they overlap or abut: adjacent query tiles)
  int jlo, jhi;
  if (na[0] == 0 && na[1] == 0) {
    jlo = jhi = 0;
  } else if (na[1] == 0) {
    jlo = ja[0]; jhi = ja[0] + na[0];
  } else if (na[0] == 0) {
    jlo = ja[1]; jhi = ja[1] + na[1];
  } else {
    jlo = min(ja[0], ja[1]);
    jhi = max(ja[0] + na[0], ja[1] + na[1]);
  }
  const int n_kv = jhi - jlo;
  auto uses = [&](int t, int j) { return j >= ja[t] && j < ja[t] + na[t]; };

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_QFULL), 1);
    mbar_init(BAR(C::B_QFULL + 1), 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(BAR(C::B_KFULL + s), 1);
      mbar_init(BAR(C::B_KEMPTY + s), 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(BAR(C::B_VFULL + s), 1);
      mbar_init(BAR(C::B_VEMPTY + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR(C::B_SFULL + t), 1);
      mbar_init(BAR(C::B_PFULL + t), 128);
      mbar_init(BAR(C::B_ODONE + t), 1);
    }
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == C::W_MMA) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::W_LOAD) {
    // ============================================================ TMA producer
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      for (int t = 0; t < 2; ++t) {
        if (na[t] == 0) continue;
        mbar_arrive_expect_tx(BAR(C::B_QFULL + t), C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(&tmQ, BAR(C::B_QFULL + t), sbase + C::OFF_Q + t * C::TILE + c * C::CHUNK,
                      c * 64, h, q_row0 + qp + t * BM, bcoord);
      }
      for (int i = 0; i < n_kv; ++i) {
        const int j = jlo + i;
        const int ks = i % KST, vs = i % VST;
        mbar_wait(BAR(C::B_KEMPTY + ks), ((uint32_t)(i / KST) & 1u) ^ 1u, abort_flag, p.status);
        mbar_arrive_expect_tx(BAR(C::B_KFULL + ks), C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(&tmK, BAR(C::B_KFULL + ks), sbase + C::OFF_K + ks * C::TILE + c * C::CHUNK,
                      c * 64, h, k_row0 + j * BN, bcoord);
        mbar_wait(BAR(C::B_VEMPTY + vs), ((uint32_t)(i / VST) & 1u) ^ 1u, abort_flag, p.status);
        mbar_arrive_expect_tx(BAR(C::B_VFULL + vs), C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(&tmV, BAR(C::B_VFULL + vs), sbase + C::OFF_V + vs * C::TILE + c * C::CHUNK,
                      c * 64, h, k_row0 + j * BN, bcoord);
      }
    }
    __syncwarp();
  } else if (warp == C::W_MMA) {
    // ============================================================ MMA issuer
    if (lane == 0 && n_kv > 0) {
      // S = Q Kᵀ: A = Q (K-major), B = K (K-major).  O += P V: A = P (tensor memory),
      // B = V stored [key][d], i.e. N-contiguous (MN-major).
      const uint32_t ID_S = idesc_f16_f32acc(BF16, BM, BN, false, false) |
                            (p.negate_scores ? (1u << 13) : 0u);  // bit 13: negate A
      constexpr uint32_t ID_O = idesc_f16_f32acc(BF16, BM, D, false, true);
      const uint64_t dQ0 = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);
      const uint64_t dK0 = sdesc_sw128(sbase + C::OFF_K, 16, 1024);
      const uint64_t dV0 = sdesc_sw128(sbase + C::OFF_V, C::CHUNK, 1024);
      int cnt[2] = {0, 0};    // S / P / O phases issued per tile
      bool qready[2] = {false, false};
      auto wait_kfull = [&](int i) {
        mbar_wait(BAR(C::B_KFULL + i % KST), (uint32_t)(i / KST) & 1u, abort_flag, p.status);
        tc_fence_after();
      };
      // S_t for key tile index i (j = jlo + i)
      auto issue_s = [&](int t, int i) {
        if (!qready[t]) {
          mbar_wait(BAR(C::B_QFULL + t), 0, abort_flag, p.status);
          tc_fence_after();
          qready[t] = true;
        }
        const uint64_t dq = sdesc_adv(dQ0, (uint32_t)(t * C::TILE));
        const uint64_t db = sdesc_adv(dK0, (uint32_t)((i % KST) * C::TILE));
        const uint32_t dst = tmem + C::TM_S + 128u * (uint32_t)t;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          mma_ss(dst, sdesc_adv(dq, off), sdesc_adv(db, off), ID_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(BAR(C::B_SFULL + t));
      };
      auto issue_pv = [&](int t, int i) {
        mbar_wait(BAR(C::B_PFULL + t), (uint32_t)cnt[t] & 1u, abort_flag, p.status);
        tc_fence_after();
        const uint64_t db = sdesc_adv(dV0, (uint32_t)((i % VST) * C::TILE));
        const uint32_t src = tmem + C::TM_S + 128u * (uint32_t)t;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(tmem + C::TM_O + (uint32_t)(t * D), src + 8u * kk, sdesc_adv(db, kk * 16 * 128),
                 ID_O, (cnt[t] > 0 || kk > 0) ? 1u : 0u);
        mma_commit(BAR(C::B_ODONE + t));
        ++cnt[t];
      };
      int k_ready = -1;  // K tiles up to this index have been waited for
      auto need_k = [&](int i) {
        if (k_ready < i) {
          wait_kfull(i);
          k_ready = i;
        }
      };
      // S of the first key tile for both query tiles
      need_k(0);
      for (int t = 0; t < 2; ++t)
        if (uses(t, jlo)) issue_s(t, 0);
      mma_commit(BAR(C::B_KEMPTY + 0));
      for (int i = 0; i < n_kv; ++i) {
        const int j = jlo + i;
        const bool next = i + 1 < n_kv;
        mbar_wait(BAR(C::B_VFULL + i % VST), (uint32_t)(i / VST) & 1u, abort_flag, p.status);
        tc_fence_after();
        // per tile: O_t += P_t V_j, then S_t of the next key tile over P_t (in order)
        for (int t = 0; t < 2; ++t) {
          if (uses(t, j)) issue_pv(t, i);
          if (next && uses(t, j + 1)) {
            need_k(i + 1);
            issue_s(t, i + 1);
          }
        }
        mma_commit(BAR(C::B_VEMPTY + i % VST));
        if (next) {
          need_k(i + 1);  // a stage is released only after its load has landed
          mma_commit(BAR(C::B_KEMPTY + (i + 1) % KST));
        }
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ============================================================ softmax warpgroups
    const int t = (warp - 4) >> 2;       // query tile of this warpgroup
    const int quarter = warp & 3;        // tensor-memory lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int q0 = qp + t * BM;
    const int i = q0 + row;              // this thread's query row
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S + 128u * (uint32_t)t;
    const uint32_t tO = tmem + lane_off + C::TM_O + (uint32_t)(t * D);
    const float c = p.scale_log2;        // > 0: scores are handled as x = s * |scale| * log2(e)
    const int n_t = na[t];
    float m = -INFINITY;                 // reference maximum of x shared by l and O
    uint64_t l2 = 0ull;                  // Σ fp32 p (paired), for the LSE
    uint64_t lr2 = 0ull;                 // Σ rounded 16-bit p (paired), normalises O

    for (int jj = 0; jj < n_t; ++jj) {
      const int j = ja[t] + jj;
      mbar_wait(BAR(C::B_SFULL + t), (uint32_t)jj & 1u, abort_flag, p.status);
      tc_fence_after();
      const int kt = j * BN;  // first key of the tile
      const bool need_mask = (kt + BN > Lk) || (wr >= 0 && kt + BN - 1 > q0 + diag + wr) ||
                             (wl >= 0 && kt < q0 + BM - 1 + diag - wl);
      // allowed columns: lo <= e < lim (only consulted when need_mask)
      const int lim = wr >= 0 ? min(Lk - kt, i + diag + wr - kt + 1) : Lk - kt;
      const int lo = wl >= 0 ? i + diag - wl - kt : 0;
      // row maximum over all 128 scores: four loads, one wait
      float mq[4];
      {
        uint32_t sr[128];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tmem_ld32(tS + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * q]));
        tmem_wait_ld();
        reg_fence(sr);
        if (need_mask) {
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e >= lim || e < lo) sr[e] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float t1[11];
#pragma unroll
          for (int e = 0; e < 10; ++e)
            t1[e] = fmax3(__uint_as_float(sr[32 * q + 3 * e]), __uint_as_float(sr[32 * q + 3 * e + 1]),
                          __uint_as_float(sr[32 * q + 3 * e + 2]));
          t1[10] = fmaxf(__uint_as_float(sr[32 * q + 30]), __uint_as_float(sr[32 * q + 31]));
          mq[q] = fmax3(fmax3(t1[0], t1[1], t1[2]), fmax3(t1[3], t1[4], t1[5]),
                        fmax3(fmax3(t1[6], t1[7], t1[8]), t1[9], t1[10]));
        }
      }
      const float mxs = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      const float mx = mxs * c;

      // Reference-maximum update: keep the stale maximum while the new one exceeds it by at
      // most 8 (a factor 2^8 in P, harmless in fp32).
      bool rescale = false;
      float alpha = 1.f;
      if (m == -INFINITY) {
        m = mx;  // first allowed keys for this row: O and the sums are still exactly 0
      } else if (mx - m > LAZY) {
        alpha = ex2_approx(m - mx);
        m = mx;
        rescale = true;
      }
      const float m_use = (m == -INFINITY) ? 0.f : m;
      const uint64_t c2 = f2_pack(c, c);
      const uint64_t nm2 = f2_pack(-m_use, -m_use);
      uint64_t ls2 = 0ull, lrs2 = 0ull;
      // kPolyPairs of every 16 pairs of exponentials run on the FMA pipe (tiles without
      // masked keys), the rest on the special-function unit
      auto exp_pass = [&](auto use_poly) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          // keys 64hh .. 64hh+63 -> packed columns 32hh .. 32hh+31; those columns belong to
          // score columns already read (the half before, or this half itself)
          uint32_t sr[64];
          tmem_ld32(tS + 64 * hh, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          tmem_ld32(tS + 64 * hh + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          tmem_wait_ld();
          reg_fence(sr);
          if (!decltype(use_poly)::value) {  // masked tiles
#pragma unroll
            for (int e = 0; e < 64; ++e)
              if (64 * hh + e >= lim || 64 * hh + e < lo) sr[e] = __float_as_uint(-INFINITY);
          }
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float2 xx = f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[32 * q + 2 * e]),
                                                         __uint_as_float(sr[32 * q + 2 * e + 1])),
                                                 c2, nm2));
              float p0, p1;
              if (decltype(use_poly)::value && e < C::kPolyPairs) {
                const float2 pp = exp2_poly2(xx.x, xx.y);
                p0 = pp.x;
                p1 = pp.y;
              } else {
                p0 = ex2_approx(xx.x);
                p1 = ex2_approx(xx.y);
              }
              pk[e] = pack2<BF16>(p0, p1);
              ls2 = f2_add(ls2, f2_pack(p0, p1));
              const float2 pr = unpack2<BF16>(pk[e]);
              lrs2 = f2_add(lrs2, f2_pack(pr.x, pr.y));
            }
            tmem_st16(tS + 32 * hh + 16 * q, pk);
          }
        }
      };
      if (need_mask)
        exp_pass(std::false_type{});
      else
        exp_pass(std::true_type{});

      if (__any_sync(0xffffffffu, rescale)) {
        // O_t was last written by the P·V product of the previous key tile: wait until it
        // completed, then rescale it in tensor memory.
        mbar_wait(BAR(C::B_ODONE + t), (uint32_t)(jj - 1) & 1u, abort_flag, p.status);
        tc_fence_after();
#pragma unroll 1
        for (int q = 0; q < D / 32; ++q) {
          uint32_t o[32];
          tmem_ld32(tO + q * 32, o);
          tmem_wait_ld();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + q * 32, o);
        }
      }
      const uint64_t a2 = f2_pack(alpha, alpha);
      l2 = f2_add(f2_mul(l2, a2), ls2);
      lr2 = f2_add(f2_mul(lr2, a2), lrs2);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(C::B_PFULL + t));
    }

    // ---------------------------------------------------------------- epilogue
    if (n_t > 0) {
      mbar_wait(BAR(C::B_ODONE + t), (uint32_t)(n_t - 1) & 1u, abort_flag, p.status);
      tc_fence_after();
    }
    const float2 lf = f2_unpack(l2), lrf = f2_unpack(lr2);
    const float L = lf.x + lf.y;
    const float LR = lrf.x + lrf.y;
    const bool valid = i < Lq;
    const float inv_l = (LR > 0.f) ? p.v_descale / LR : 0.f;
    const size_t orow_idx = (p.cu_q != nullptr) ? ((size_t)(q_row0 + i) * p.H + h) * D
                                                : (((size_t)bcoord * p.N + i) * p.H + h) * D;
#pragma unroll 1
    for (int q = 0; q < D / 32; ++q) {
      uint32_t o[32];
      if (n_t > 0) {
        tmem_ld32(tO + q * 32, o);
        tmem_wait_ld();
        reg_fence(o);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (!valid) continue;
      if constexpr (F32O) {
        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.o) + orow_idx + q * 32);
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4)
          dst[v4] = make_float4(__uint_as_float(o[4 * v4]) * inv_l, __uint_as_float(o[4 * v4 + 1]) * inv_l,
                                __uint_as_float(o[4 * v4 + 2]) * inv_l, __uint_as_float(o[4 * v4 + 3]) * inv_l);
      } else {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack2<BF16>(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.o) + orow_idx + q * 32);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
      }
    }
    if (valid) {
      const float lse = (L > 0.f) ? (m + lg2_approx(L)) * 0.69314718055994530942f : INFINITY;
      if (p.cu_q != nullptr)
        p.lse[(size_t)h * p.total_q + q_row0 + i] = lse;
      else
        p.lse[((size_t)bcoord * p.H + h) * p.N + i] = lse;
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == C::W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fattn
