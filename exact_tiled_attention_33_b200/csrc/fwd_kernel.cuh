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
//   * one CTA owns QT = 2 query tiles of BM = 128 rows and walks the key/value tiles
//     (BN = 128 keys) that any of its rows may see; both query tiles share each K/V tile;
//   * warp 0 issues TMA loads (Q once; K and V through a STAGES-deep ring);
//   * warp 1, one thread, issues tcgen05.mma: S_t = Q_t K_jᵀ into tensor memory
//     (shared x shared), and O_t += P_t V_j with P_t read from tensor memory;
//   * warps 4..11 form two softmax warpgroups, one per query tile; thread r of a group
//     owns row r (= tensor-memory lane r): it reads its row of S with tcgen05.ld, masks,
//     updates m and l in the exp2 domain, writes P back over S as packed 16-bit values,
//     and rescales its row of O only when the row maximum grew by more than 2^8
//     (exact: O and l always share the same reference maximum);
//   * tensor memory: S0 | S1 | O0 | O1 (128 + 128 + D + D columns of 32 bits).
#pragma once

#include <type_traits>

#include "fattn_internal.h"
#include "sm100.cuh"

namespace fattn {

template <int D>
struct FwdCfg {
  static constexpr int BM = 128;  // query rows per tile = tensor-memory lanes
  static constexpr int BN = 128;  // keys per K/V tile
  static constexpr int QT = 2;    // query tiles per CTA
  static constexpr int STAGES = (D == 128) ? 2 : 4;
  static constexpr int KCH = D / 64;  // 128-byte (64-element) column chunks per row
  static constexpr int Q_CHUNK = BM * 128;
  static constexpr int KV_CHUNK = BN * 128;
  static constexpr int Q_TILE = BM * D * 2;
  static constexpr int KV_TILE = BN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QT * Q_TILE;
  static constexpr int OFF_V = OFF_K + STAGES * KV_TILE;
  static constexpr int OFF_BAR = OFF_V + STAGES * KV_TILE;
  // barriers
  static constexpr int B_QFULL = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_KEMPTY = B_KFULL + STAGES;
  static constexpr int B_VFULL = B_KEMPTY + STAGES;
  static constexpr int B_VEMPTY = B_VFULL + STAGES;
  static constexpr int B_SFULL = B_VEMPTY + STAGES;
  static constexpr int B_PFULL = B_SFULL + QT;
  static constexpr int B_OFULL = B_PFULL + QT;
  static constexpr int NBAR = B_OFULL + QT;
  static constexpr int SMEM_BYTES = OFF_BAR + 8 * NBAR + 16 + 1024;  // + alignment slack
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  // 12 warps: warpgroup 0 = {loads, MMA, 2 idle}, warpgroups 1 and 2 = softmax for query
  // tiles 0 and 1.  Registers move from warpgroup 0 to the softmax warpgroups:
  // 128 x 112 + 256 x 192 = 63488 <= 384 x 168 (the launch allocation); with these
  // neither the MMA issuer nor the softmax (128 scores per thread) spills.
  static constexpr int THREADS = 384;
  static constexpr uint32_t REGS_LOAD = 112, REGS_SOFTMAX = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  // pairs of every 16 (per 32-column chunk) whose exponentials use exp2_poly2
  static constexpr int kPolyPairs = 4;
  // tensor-memory column of S_t (P_t aliases its first BN/2 columns) and of O_t
  __device__ static constexpr uint32_t tm_s(int t) { return (uint32_t)t * 128u; }
  __device__ static constexpr uint32_t tm_o(int t) { return 256u + (uint32_t)t * D; }
};

template <int D, bool BF16>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<D>;
  constexpr int BM = C::BM, BN = C::BN, QT = C::QT, ST = C::STAGES;

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
  // grid: x = query-tile pair (fastest, so the CTAs running together share one head's
  // K/V in L2), y = head, z = batch or sequence; when causal the pair with the most key
  // tiles of each head is launched first.
  const int h = blockIdx.y;
  const int bz = blockIdx.z;
  const int pair = p.causal ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
  int Lq, Lk, q_row0, k_row0, bcoord;
  if (p.cu_q != nullptr) {
    const int s = bz;
    q_row0 = p.cu_q[s];
    Lq = p.cu_q[s + 1] - q_row0;
    k_row0 = p.cu_k[s];
    Lk = p.cu_k[s + 1] - k_row0;
    bcoord = 0;
  } else {
    q_row0 = 0;
    k_row0 = 0;
    Lq = Lk = p.N;
    bcoord = bz;
  }
  const int q0 = pair * (BM * QT);
  if (q0 >= Lq) return;  // uniform for the whole CTA
  const int diag = Lk - Lq;  // key j is allowed for row i iff j <= i + diag (causal)
  const int kv_tiles_all = (Lk + BN - 1) / BN;
  int n_kv = kv_tiles_all;
  if (p.causal) {
    const int r_last = min(q0 + BM * QT - 1, Lq - 1);
    const int j_last = r_last + diag;
    n_kv = (j_last < 0) ? 0 : min(kv_tiles_all, j_last / BN + 1);
  }

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_QFULL), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(BAR(C::B_KFULL + s), 1);
      mbar_init(BAR(C::B_KEMPTY + s), 1);
      mbar_init(BAR(C::B_VFULL + s), 1);
      mbar_init(BAR(C::B_VEMPTY + s), 1);
    }
    for (int t = 0; t < QT; ++t) {
      mbar_init(BAR(C::B_SFULL + t), 1);
      mbar_init(BAR(C::B_PFULL + t), BM);
      mbar_init(BAR(C::B_OFULL + t), 1);
    }
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
   regs_dealloc<C::REGS_LOAD>();
   if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(BAR(C::B_QFULL), QT * C::Q_TILE);
      for (int t = 0; t < QT; ++t)
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(&tmQ, BAR(C::B_QFULL),
                      sbase + C::OFF_Q + t * C::Q_TILE + c * C::Q_CHUNK, c * 64, h,
                      q_row0 + q0 + t * BM, bcoord);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % ST;
        const uint32_t ph = (uint32_t)(j / ST) & 1u;
        mbar_wait(BAR(C::B_KEMPTY + s), ph ^ 1u, abort_flag, p.status);
        mbar_arrive_expect_tx(BAR(C::B_KFULL + s), C::KV_TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(&tmK, BAR(C::B_KFULL + s), sbase + C::OFF_K + s * C::KV_TILE + c * C::KV_CHUNK,
                      c * 64, h, k_row0 + j * BN, bcoord);
        mbar_wait(BAR(C::B_VEMPTY + s), ph ^ 1u, abort_flag, p.status);
        mbar_arrive_expect_tx(BAR(C::B_VFULL + s), C::KV_TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(&tmV, BAR(C::B_VFULL + s), sbase + C::OFF_V + s * C::KV_TILE + c * C::KV_CHUNK,
                      c * 64, h, k_row0 + j * BN, bcoord);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0 && n_kv > 0) {
      // S = Q Kᵀ: A = Q (K-major), B = K (K-major).  O += P V: A = P (tensor memory),
      // B = V stored [key][d], i.e. N-contiguous (MN-major).
      const uint32_t ID_S = idesc_f16_f32acc(BF16, BM, BN, false, false) |
                            (p.negate_scores ? (1u << 13) : 0u);  // bit 13: negate A
      constexpr uint32_t ID_O = idesc_f16_f32acc(BF16, BM, D, false, true);
      // Descriptors built once; each MMA only adds a compile-time offset.
      const uint64_t dQ0 = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);
      const uint64_t dK0 = sdesc_sw128(sbase + C::OFF_K, 16, 1024);
      const uint64_t dV0 = sdesc_sw128(sbase + C::OFF_V, C::KV_CHUNK, 1024);
      auto issue_s = [&](int t, int s) {
        const uint64_t da = sdesc_adv(dQ0, (uint32_t)(t * C::Q_TILE));
        const uint64_t db = sdesc_adv(dK0, (uint32_t)(s * C::KV_TILE));
        const uint32_t dst = tmem + C::tm_s(t);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(dst, sdesc_adv(da, (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32),
                 sdesc_adv(db, (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32), ID_S, kk > 0 ? 1u : 0u);
      };
      auto issue_pv = [&](int t, int s, bool accumulate) {
        const uint64_t db = sdesc_adv(dV0, (uint32_t)(s * C::KV_TILE));
        const uint32_t dst = tmem + C::tm_o(t), src = tmem + C::tm_s(t);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(dst, src + kk * 8, sdesc_adv(db, kk * 16 * 128), ID_O,
                 (accumulate || kk > 0) ? 1u : 0u);
      };
      mbar_wait(BAR(C::B_QFULL), 0, abort_flag, p.status);
      tc_fence_after();
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % ST;
        mbar_wait(BAR(C::B_KFULL + s), (uint32_t)(j / ST) & 1u, abort_flag, p.status);
        tc_fence_after();
        for (int t = 0; t < QT; ++t) {
          if (j > 0) {
            const int ps = (j - 1) % ST;
            mbar_wait(BAR(C::B_PFULL + t), (uint32_t)(j - 1) & 1u, abort_flag, p.status);
            if (t == 0) mbar_wait(BAR(C::B_VFULL + ps), (uint32_t)((j - 1) / ST) & 1u, abort_flag, p.status);
            tc_fence_after();
            issue_pv(t, ps, j - 1 > 0);
            if (t == QT - 1) mma_commit(BAR(C::B_VEMPTY + ps));
          }
          // S_t is overwritten only after the P_t it holds was consumed by the P·V
          // product issued just above (tcgen05.mma from one thread run in order).
          issue_s(t, s);
          mma_commit(BAR(C::B_SFULL + t));
        }
        mma_commit(BAR(C::B_KEMPTY + s));
      }
      const int jl = n_kv - 1;
      const int ls = jl % ST;
      for (int t = 0; t < QT; ++t) {
        mbar_wait(BAR(C::B_PFULL + t), (uint32_t)jl & 1u, abort_flag, p.status);
        if (t == 0) mbar_wait(BAR(C::B_VFULL + ls), (uint32_t)(jl / ST) & 1u, abort_flag, p.status);
        tc_fence_after();
        issue_pv(t, ls, jl > 0);
        mma_commit(BAR(C::B_OFULL + t));
        if (t == QT - 1) mma_commit(BAR(C::B_VEMPTY + ls));
      }
    }
    __syncwarp();
   }
  } else {
    regs_alloc<C::REGS_SOFTMAX>();
    // ============================================================ softmax warpgroups
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;  // tensor-memory lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int r0 = q0 + t * BM;  // first query row of this tile (within the sequence)
    const int i = r0 + row;      // this thread's query row
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::tm_s(t);
    const uint32_t tO = tmem + lane_off + C::tm_o(t);
    const float c = p.scale_log2;  // > 0: scores are handled as x = s * scale * log2(e)
    float m = -INFINITY;           // reference maximum of x shared by l and O
    float l = 0.f;                 // Σ p (fp32), for the log-sum-exp
    float l_r = 0.f;               // Σ of the 16-bit P actually multiplied into O

    for (int j = 0; j < n_kv; ++j) {
      mbar_wait(BAR(C::B_SFULL + t), (uint32_t)j & 1u, abort_flag, p.status);
      tc_fence_after();
      // Raw scores s; the scaled, log2-domain score is x = s * c with c > 0 (a negative
      // softmax scale is applied by negating Q inside the S product).
      uint32_t sr[128];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[q * 32]));
      tmem_wait_ld();
      reg_fence(sr);

      const int k0 = j * BN;
      const bool need_mask = (k0 + BN > Lk) || (p.causal && (k0 + BN - 1 > r0 + diag));
      if (need_mask) {
        int lim = Lk - k0;  // keys k0 + e with e < lim are allowed
        if (p.causal) lim = min(lim, i + diag - k0 + 1);
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (e >= lim) sr[e] = __float_as_uint(-INFINITY);
      }
      // Row maximum as a tree of 3-input maxima (depth 5 instead of a 64-long chain).
      float t1[43];
#pragma unroll
      for (int e = 0; e < 42; ++e)
        t1[e] = fmax3(__uint_as_float(sr[3 * e]), __uint_as_float(sr[3 * e + 1]),
                      __uint_as_float(sr[3 * e + 2]));
      t1[42] = fmaxf(__uint_as_float(sr[126]), __uint_as_float(sr[127]));
      float t2[15];
#pragma unroll
      for (int e = 0; e < 14; ++e) t2[e] = fmax3(t1[3 * e], t1[3 * e + 1], t1[3 * e + 2]);
      t2[14] = t1[42];
      const float t3a = fmax3(t2[0], t2[1], t2[2]), t3b = fmax3(t2[3], t2[4], t2[5]);
      const float t3c = fmax3(t2[6], t2[7], t2[8]), t3d = fmax3(t2[9], t2[10], t2[11]);
      const float t3e = fmax3(t2[12], t2[13], t2[14]);
      const float mx = fmax3(fmax3(t3a, t3b, t3c), t3d, t3e) * c;

      // Reference-maximum update.  Keep the stale maximum while the new one exceeds
      // it by at most 8 (a factor 2^8 in P, harmless in fp32 accumulators).
      bool rescale = false;
      float alpha = 1.f;
      if (m == -INFINITY) {
        m = mx;  // first allowed keys for this row: O and l are still exactly 0
      } else if (mx - m > 8.f) {
        alpha = ex2_approx(m - mx);
        m = mx;
        rescale = true;
      }
      const float m_use = (m == -INFINITY) ? 0.f : m;
      // p = 2^(s*c - m).  Two sums: l (exact fp32 p) gives the log-sum-exp; lr sums the
      // 16-bit values the P·V product actually uses and normalises O, so numerator and
      // denominator share the rounding of P (with the lazy maximum the largest P of a
      // row is 2^δ, not exactly 1, and its rounding would otherwise bias the output).
      const uint64_t c2 = f2_pack(c, c);
      const uint64_t nm2 = f2_pack(-m_use, -m_use);
      uint64_t ls2 = 0ull, lr2 = 0ull;
      // A quarter of the exponentials run on the FMA pipe (tiles without masked keys), the
      // rest on the special-function unit, so that both units finish within the time of
      // the tile's two matrix products.  The choice is made once per tile: the loop
      // bodies stay branch-free.
      auto exp_pass = [&](auto use_poly) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t pk[16];
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
            pk[e] = pack2<BF16>(p0, p1);
            const float2 pr = unpack2<BF16>(pk[e]);
            ls2 = f2_add(ls2, f2_pack(p0, p1));
            lr2 = f2_add(lr2, f2_pack(pr.x, pr.y));
          }
          tmem_st16(tS + q * 16, pk);
        }
      };
      if (need_mask)
        exp_pass(std::false_type{});
      else
        exp_pass(std::true_type{});
      const float2 ls = f2_unpack(ls2), lr = f2_unpack(lr2);
      l = l * alpha + (ls.x + ls.y);
      l_r = l_r * alpha + (lr.x + lr.y);

      if (__any_sync(0xffffffffu, rescale)) {
        // O_t was last written by the P·V product of tile j-1, which completed before
        // S_t of tile j was signalled, so it is stable here.
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
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(C::B_PFULL + t));
    }

    // ---------------------------------------------------------------- epilogue
    if (n_kv > 0) {
      mbar_wait(BAR(C::B_OFULL + t), 0, abort_flag, p.status);
      tc_fence_after();
    }
    const bool valid = i < Lq;
    const float inv_l = (l_r > 0.f) ? 1.f / l_r : 0.f;
    using elem_t = uint16_t;
    elem_t* orow;
    if (p.cu_q != nullptr)
      orow = reinterpret_cast<elem_t*>(p.o) + ((size_t)(q_row0 + i) * p.H + h) * D;
    else
      orow = reinterpret_cast<elem_t*>(p.o) + (((size_t)bcoord * p.N + i) * p.H + h) * D;
#pragma unroll 1
    for (int q = 0; q < D / 32; ++q) {
      uint32_t o[32];
      if (n_kv > 0) {
        tmem_ld32(tO + q * 32, o);
        tmem_wait_ld();
        reg_fence(o);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pk[e] = pack2<BF16>(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
      }
    }
    if (valid) {
      const float lse = (l > 0.f) ? (m + lg2_approx(l)) * 0.69314718055994530942f : INFINITY;
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
