// Backward pass of exact attention for sm_100a: recompute P from Q, K and the saved
// log-sum-exp, then accumulate dV, dK per key tile and dQ across key tiles.
//
// Method (what is computed): the backward pass recomputes the forward path instead of
// storing the N×N matrix (page "Flash Attention V3：大模型训练加速与显存优化技术解析" §3.2:
// recomputation, O(N) storage, global gradients split into local updates).  With
// D_i = Σ_c dO_ic O_ic and P_ij = exp(scale q_i·k_j − LSE_i):
//   dV_j = Σ_i P_ij dO_i,   dP_ij = dO_i·v_j,   dS_ij = P_ij (dP_ij − D_i),
//   dK_j = scale Σ_i dS_ij q_i,   dQ_i = scale Σ_j dS_ij k_j,
// the chain rule applied to the "standard attention" definition of the page
// "FlashAttention-2的核心设计原理".
//
// Kernels (the "global gradients split into local updates" of the same page, read as
// two independent passes so that no gradient is ever accumulated across CTAs):
//   fa_bwd_pre_kernel   D = rowsum(dO ∘ O), one warp per row, warp-shuffle reduction
//   fa_bwd_dkdv_kernel  one CTA per 128-key tile, looping over the query tiles that can
//                       see it: Sᵀ = K Qᵀ, dPᵀ = V dOᵀ, dV += Pᵀ dO, dK += dSᵀ Q
//   fa_bwd_dq_kernel    one CTA per 128-row query tile, looping over the key tiles it
//                       can see: S = Q Kᵀ, dP = dO Vᵀ, dQ += dS K
// P and dS are recomputed in both (7 products instead of 5) in exchange for no fp32
// atomics at all: every output element is written exactly once, so dQ, dK and dV are
// bitwise reproducible.  All products run on tcgen05 with fp32 accumulators in tensor
// memory; P and dS re-enter the tensor core from tensor memory (packed 16-bit).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fattn_internal.h"
#include "sm100.cuh"

namespace fattn {

// ------------------------------------------------------------------ preprocess
// One warp per (row, head) of O / dO.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const BwdParams p, long long rows_total) {
  constexpr int PER = D / 32;  // elements per lane
  const long long warps = (long long)gridDim.x * (blockDim.x / 32);
  const int lane = threadIdx.x & 31;
  for (long long w = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); w < rows_total * p.H;
       w += warps) {
    const long long row = w / p.H;  // token row (b*N + n, or packed index)
    const int h = (int)(w - row * p.H);
    const size_t base = (size_t)w * D + lane * PER;
    const uint16_t* o = reinterpret_cast<const uint16_t*>(p.o) + base;
    const uint16_t* g = reinterpret_cast<const uint16_t*>(p.dout) + base;
    float acc = 0.f;
    if constexpr (PER == 4) {
      const uint2 a = *reinterpret_cast<const uint2*>(o);
      const uint2 b = *reinterpret_cast<const uint2*>(g);
      const uint32_t av[2] = {a.x, a.y}, bv[2] = {b.x, b.y};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float2 fa, fb;
        if constexpr (BF16) {
          fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[e]));
          fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[e]));
        } else {
          fa = __half22float2(*reinterpret_cast<const __half2*>(&av[e]));
          fb = __half22float2(*reinterpret_cast<const __half2*>(&bv[e]));
        }
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
    } else {
      const uint32_t a = *reinterpret_cast<const uint32_t*>(o);
      const uint32_t b = *reinterpret_cast<const uint32_t*>(g);
      float2 fa, fb;
      if constexpr (BF16) {
        fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a));
        fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b));
      } else {
        fa = __half22float2(*reinterpret_cast<const __half2*>(&a));
        fb = __half22float2(*reinterpret_cast<const __half2*>(&b));
      }
      acc = fmaf(fa.x, fb.x, fmaf(fa.y, fb.y, acc));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      size_t di;
      if (p.cu_q != nullptr) {
        di = (size_t)h * p.total_q + row;
      } else {
        const long long b = row / p.N, n = row - b * p.N;
        di = ((size_t)b * p.H + h) * p.N + n;
      }
      p.dvec[di] = acc;
    }
  }
}

// ------------------------------------------------------------------ shared layout
template <int D>
struct BwdCfg {
  static constexpr int BM = 128;  // query rows per tile
  static constexpr int BN = 128;  // keys per tile
  static constexpr int STAGES = 2;
  static constexpr int KCH = D / 64;
  static constexpr int CHUNK = 128 * 128;  // one 64-column chunk of a 128-row tile
  static constexpr int TILE = 128 * D * 2;
  // dK/dV kernel: K, V resident; Q and dO streamed with per-tile vectors
  static constexpr int A_OFF_K = 0;
  static constexpr int A_OFF_V = A_OFF_K + TILE;
  static constexpr int A_OFF_Q = A_OFF_V + TILE;
  static constexpr int A_OFF_DO = A_OFF_Q + STAGES * TILE;
  static constexpr int A_OFF_VEC = A_OFF_DO + STAGES * TILE;  // per stage: -lse*log2e, D
  static constexpr int A_OFF_BAR = A_OFF_VEC + STAGES * 2 * BM * 4;
  // dQ kernel: Q and dO resident in tensor memory (the A operands of S and dP); K streamed
  // through 3 stages (it is needed from the S product one step ahead until the dQ
  // product), V through 3
  static constexpr int K_STAGES = 3;
  static constexpr int V_STAGES = 3;
  static constexpr int B_OFF_K = 0;
  static constexpr int B_OFF_V = B_OFF_K + K_STAGES * TILE;
  static constexpr int B_OFF_BAR = B_OFF_V + V_STAGES * TILE;
  static constexpr int NBAR = 24;  // mbarrier slots reserved in either kernel
  static constexpr int SMEM_A = A_OFF_BAR + 8 * NBAR + 16 + 1024;
  static constexpr int SMEM_B = B_OFF_BAR + 8 * NBAR + 16 + 1024;
  static_assert(SMEM_A <= 232448 && SMEM_B <= 232448, "shared memory per CTA");
  static constexpr int THREADS = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  // packed 16-bit operand column for K-elements 16*kk .. 16*kk+15 of a 128-wide row:
  // half 0 (elements 0..63) packs into columns 0..31, half 1 into 64..95 of its region
  __device__ static constexpr uint32_t packed_col(int kk) {
    return (uint32_t)(kk * 8 + (kk >= 4 ? 32 : 0));
  }
};

// Roles (12 warps): 0 loads, 1 issues MMAs, 2-3 idle, 4-7 and 8-11 are two compute
// warpgroups, each owning half of the 128 columns of every score tile (one tensor-memory
// lane = one row per thread).

// ------------------------------------------------------------------ dK, dV
// Tensor memory: Sᵀ [0,128) (Pᵀ packed into it) | dPᵀ [128,256) (dSᵀ packed into it) |
// dK [256, 256+D) | dV [256+D, 256+2D).
// Grid: x = key tile (fastest, so the CTAs running together share one head's Q/dO in
// L2; tile 0, which has the most query tiles when causal, first), y = head, z = batch or
// sequence.
template <int D, bool BF16>
__global__ void __launch_bounds__(384, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int BM = C::BM, BN = C::BN, ST = C::STAGES;
  constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DK = 256, TM_DV = 256 + D;
  enum { B_KV = 0, B_QFULL = 1, B_QEMPTY = B_QFULL + ST, B_SFULL = B_QEMPTY + ST, B_DPFULL,
         B_PFULL, B_DSFULL, B_DONE };
  static_assert(B_DONE < C::NBAR, "mbarrier slots");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::A_OFF_BAR + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + C::A_OFF_BAR + 8 * C::NBAR);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int h = blockIdx.y;
  const int bz = blockIdx.z;
  int Lq, Lk, q_row0, k_row0, bcoord;
  if (p.cu_q != nullptr) {
    if (!varlen_segment_ok(p.cu_q, p.cu_k, bz, p.total_q, p.total_k, -1, p.max_seqlen_k,
                           p.status))
      return;
    q_row0 = p.cu_q[bz];
    Lq = p.cu_q[bz + 1] - q_row0;
    k_row0 = p.cu_k[bz];
    Lk = p.cu_k[bz + 1] - k_row0;
    bcoord = 0;
  } else {
    q_row0 = k_row0 = 0;
    Lq = Lk = p.N;
    bcoord = bz;
  }
  const int k0 = blockIdx.x * BN;
  if (k0 >= Lk) return;
  const int diag = Lk - Lq;  // bottom-right alignment of the window (causal: j <= i + diag)
  const int wl = p.win_left, wr = p.win_right;
  int i_begin, n_q;          // query tiles i_begin .. i_begin + n_q - 1
  query_tile_range(k0, min(k0 + BN - 1, Lk - 1), Lq, diag, wl, wr, BM, &i_begin, &n_q);

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_KV), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(BAR(B_QFULL + s), 32);
      mbar_init(BAR(B_QEMPTY + s), 1);
    }
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_DPFULL), 1);
    mbar_init(BAR(B_PFULL), 256);
    mbar_init(BAR(B_DSFULL), 256);
    mbar_init(BAR(B_DONE), 1);
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
  const float kLog2e = 1.4426950408889634f;

  if (warp == 0) {
    // ============================================================ loads
    if (n_q > 0) {
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmDO);
        mbar_arrive_expect_tx(BAR(B_KV), 2 * C::TILE);
        for (int c = 0; c < C::KCH; ++c) {
          tma_load_4d(&tmK, BAR(B_KV), sbase + C::A_OFF_K + c * C::CHUNK, c * 64, h, k_row0 + k0,
                      bcoord);
          tma_load_4d(&tmV, BAR(B_KV), sbase + C::A_OFF_V + c * C::CHUNK, c * 64, h, k_row0 + k0,
                      bcoord);
        }
      }
      for (int it = 0; it < n_q; ++it) {
        const int s = it % ST;
        const int q0 = (i_begin + it) * BM;
        mbar_wait(BAR(B_QEMPTY + s), ((uint32_t)(it / ST) & 1u) ^ 1u, abort_flag, p.status);
        // -LSE·log2(e) and D of the 128 query rows; rows past the sequence: -inf, 0.
        float* vec = reinterpret_cast<float*>(sgen + C::A_OFF_VEC + s * 2 * BM * 4);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qc = lane * 4 + e;
          const int qg = q0 + qc;
          float nl2 = -INFINITY, dd = 0.f;
          if (qg < Lq) {
            const size_t vi = (p.cu_q != nullptr) ? (size_t)h * p.total_q + q_row0 + qg
                                                  : ((size_t)bcoord * p.H + h) * p.N + qg;
            nl2 = -p.lse[vi] * kLog2e;
            dd = p.dvec[vi];
          }
          vec[qc] = nl2;
          vec[BM + qc] = dd;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(BAR(B_QFULL + s), 2 * C::TILE);
          for (int c = 0; c < C::KCH; ++c) {
            tma_load_4d(&tmQ, BAR(B_QFULL + s), sbase + C::A_OFF_Q + s * C::TILE + c * C::CHUNK,
                        c * 64, h, q_row0 + q0, bcoord);
            tma_load_4d(&tmDO, BAR(B_QFULL + s), sbase + C::A_OFF_DO + s * C::TILE + c * C::CHUNK,
                        c * 64, h, q_row0 + q0, bcoord);
          }
        } else {
          mbar_arrive(BAR(B_QFULL + s));
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0 && n_q > 0) {
      constexpr uint32_t ID_ST = idesc_f16_f32acc(BF16, 128, 128, false, false);  // Sᵀ, dPᵀ
      constexpr uint32_t ID_ACC = idesc_f16_f32acc(BF16, 128, D, false, true);    // dV, dK
      // Descriptors built once; each MMA only adds a compile-time offset.
      const uint64_t dK = sdesc_sw128(sbase + C::A_OFF_K, 16, 1024);
      const uint64_t dV = sdesc_sw128(sbase + C::A_OFF_V, 16, 1024);
      const uint64_t dQk = sdesc_sw128(sbase + C::A_OFF_Q, 16, 1024);          // K-major
      const uint64_t dDOk = sdesc_sw128(sbase + C::A_OFF_DO, 16, 1024);        // K-major
      const uint64_t dQm = sdesc_sw128(sbase + C::A_OFF_Q, C::CHUNK, 1024);    // MN-major
      const uint64_t dDOm = sdesc_sw128(sbase + C::A_OFF_DO, C::CHUNK, 1024);  // MN-major
      // X = A Bᵀ with A = [keys][d] (K-major) and B = [queries][d] (K-major)
      auto issue_kt = [&](uint32_t dst, uint64_t da, uint64_t db) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          mma_ss(tmem + dst, sdesc_adv(da, off), sdesc_adv(db, off), ID_ST, kk > 0 ? 1u : 0u);
        }
      };
      // Acc += Xᵀ-packed (tensor memory, keys x queries) · B with B = [queries][d]
      auto issue_acc = [&](uint32_t acc, uint32_t src, uint64_t db, bool accumulate) {
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          mma_ts(tmem + acc, tmem + src + C::packed_col(kk), sdesc_adv(db, kk * 2048), ID_ACC,
                 (accumulate || kk > 0) ? 1u : 0u);
      };
      auto wait_q = [&](int it) {
        mbar_wait(BAR(B_QFULL + it % ST), (uint32_t)(it / ST) & 1u, abort_flag, p.status);
        tc_fence_after();
      };
      mbar_wait(BAR(B_KV), 0, abort_flag, p.status);
      wait_q(0);
      issue_kt(TM_S, dK, dQk);
      mma_commit(BAR(B_SFULL));
      issue_kt(TM_DP, dV, dDOk);
      mma_commit(BAR(B_DPFULL));
      for (int it = 0; it < n_q; ++it) {
        const int s = it % ST;
        const int s1 = (it + 1) % ST;
        const uint32_t ph = (uint32_t)it & 1u;
        mbar_wait(BAR(B_PFULL), ph, abort_flag, p.status);
        tc_fence_after();
        issue_acc(TM_DV, TM_S, sdesc_adv(dDOm, s * C::TILE), it > 0);   // dV += Pᵀ dO
        if (it + 1 < n_q) {                          // Sᵀ of the next step over Pᵀ
          wait_q(it + 1);
          issue_kt(TM_S, dK, sdesc_adv(dQk, s1 * C::TILE));
          mma_commit(BAR(B_SFULL));
        }
        mbar_wait(BAR(B_DSFULL), ph, abort_flag, p.status);
        tc_fence_after();
        issue_acc(TM_DK, TM_DP, sdesc_adv(dQm, s * C::TILE), it > 0);   // dK += dSᵀ Q
        mma_commit(BAR(B_QEMPTY + s));
        if (it + 1 < n_q) {                          // dPᵀ of the next step over dSᵀ
          issue_kt(TM_DP, dV, sdesc_adv(dDOk, s1 * C::TILE));
          mma_commit(BAR(B_DPFULL));
        }
      }
      mma_commit(BAR(B_DONE));
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ============================================================ compute: Pᵀ, dSᵀ
    const int half = (warp - 4) >> 2;   // query columns 64*half .. 64*half+63
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row within the tile
    const int kg = k0 + r;              // key index within the sequence
    const bool key_ok = kg < Lk;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + TM_S + 64 * half;
    const uint32_t tDP = tmem + lane_off + TM_DP + 64 * half;
    const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
    const int cbase = 64 * half;
    for (int it = 0; it < n_q; ++it) {
      const int s = it % ST;
      const uint32_t ph = (uint32_t)it & 1u;
      const int q0 = (i_begin + it) * BM;
      const float* vec = reinterpret_cast<const float*>(sgen + C::A_OFF_VEC + s * 2 * BM * 4);
      const bool need_mask = (k0 + BN > Lk) || (q0 + BM > Lq) ||
                             (wr >= 0 && k0 + BN - 1 > q0 + diag + wr) ||
                             (wl >= 0 && k0 < q0 + BM - 1 + diag - wl);
      // allowed columns (query q0 + c): qmin <= c < qend
      const int qmin = wr >= 0 ? kg - diag - wr - q0 : -1;
      const int qend = wl >= 0 ? min(Lq - q0, kg - diag + wl - q0 + 1) : Lq - q0;
      mbar_wait(BAR(B_QFULL + s), (uint32_t)(it / ST) & 1u, abort_flag, p.status);
      mbar_wait(BAR(B_SFULL), ph, abort_flag, p.status);
      tc_fence_after();
      uint32_t sv[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_wait_ld();
      reg_fence(sv);
      // p = 2^(s*c - LSE*log2e): one branch-free pass (so the exp latency of different
      // columns overlaps), masks applied afterwards only on boundary tiles.
      const float4* nl4 = reinterpret_cast<const float4*>(&vec[cbase]);
      float pv[64];
#pragma unroll
      for (int e4 = 0; e4 < 16; ++e4) {
        const float4 nl = nl4[e4];
        const float2 x0 = f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[4 * e4]), __uint_as_float(sv[4 * e4 + 1])),
                                           c2, f2_pack(nl.x, nl.y)));
        const float2 x1 = f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[4 * e4 + 2]), __uint_as_float(sv[4 * e4 + 3])),
                                           c2, f2_pack(nl.z, nl.w)));
        pv[4 * e4] = ex2_approx(x0.x);
        pv[4 * e4 + 1] = ex2_approx(x0.y);
        pv[4 * e4 + 2] = ex2_approx(x1.x);
        pv[4 * e4 + 3] = ex2_approx(x1.y);
      }
      if (need_mask) {
        // allowed columns c: key in range, qmin <= c < qend (window and sequence end)
        const int lo = key_ok ? max(qmin, 0) - cbase : 64;
        const int hi = min(qend, 128) - cbase;
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (e < lo || e >= hi) pv[e] = 0.f;
      }
      uint32_t pk[32];  // Pᵀ row segment, packed 16-bit pairs
#pragma unroll
      for (int e = 0; e < 32; ++e) pk[e] = pack2<BF16>(pv[2 * e], pv[2 * e + 1]);
      tmem_st32(tS, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(B_PFULL));

      // dSᵀ = Pᵀ ∘ (dPᵀ − D), packed over this thread's own dPᵀ columns.
      mbar_wait(BAR(B_DPFULL), ph, abort_flag, p.status);
      tc_fence_after();
      uint32_t dv[64];
      tmem_ld32(tDP, *reinterpret_cast<uint32_t(*)[32]>(&dv[0]));
      tmem_ld32(tDP + 32, *reinterpret_cast<uint32_t(*)[32]>(&dv[32]));
      tmem_wait_ld();
      reg_fence(dv);
      const float4* d4 = reinterpret_cast<const float4*>(&vec[BM + cbase]);
      uint32_t ds[32];
#pragma unroll
      for (int e4 = 0; e4 < 16; ++e4) {
        const float4 dd = d4[e4];
        const float2 pa = unpack2<BF16>(pk[2 * e4]);
        const float2 pb = unpack2<BF16>(pk[2 * e4 + 1]);
        const float2 da = f2_unpack(f2_mul(f2_add(f2_pack(__uint_as_float(dv[4 * e4]), __uint_as_float(dv[4 * e4 + 1])),
                                                  f2_pack(-dd.x, -dd.y)),
                                           f2_pack(pa.x, pa.y)));
        const float2 db = f2_unpack(f2_mul(f2_add(f2_pack(__uint_as_float(dv[4 * e4 + 2]), __uint_as_float(dv[4 * e4 + 3])),
                                                  f2_pack(-dd.z, -dd.w)),
                                           f2_pack(pb.x, pb.y)));
        ds[2 * e4] = pack2<BF16>(da.x, da.y);
        ds[2 * e4 + 1] = pack2<BF16>(db.x, db.y);
      }
      tmem_st32(tDP, ds);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(B_DSFULL));
    }
    // ---------------------------------------------------------------- epilogue
    // half 0 stores dV, half 1 stores dK = scale · Σ dSᵀ Q
    if (n_q > 0) {
      mbar_wait(BAR(B_DONE), 0, abort_flag, p.status);
      tc_fence_after();
    }
    uint16_t* orow = reinterpret_cast<uint16_t*>(half == 0 ? p.dv : p.dk) +
                     (p.cu_q != nullptr ? ((size_t)(k_row0 + kg) * p.H + h) * D
                                        : (((size_t)bcoord * p.N + kg) * p.H + h) * D);
    const float sc = half == 0 ? 1.f : p.scale;
    const uint32_t tsrc = tmem + lane_off + (half == 0 ? TM_DV : TM_DK);
#pragma unroll 1
    for (int q = 0; q < D / 32; ++q) {
      uint32_t v[32];
      if (n_q > 0) {
        tmem_ld32(tsrc + q * 32, v);
        tmem_wait_ld();
        reg_fence(v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if (key_ok) {
        uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          dst[u] = make_uint4(
              pack2<BF16>(__uint_as_float(v[8 * u]) * sc, __uint_as_float(v[8 * u + 1]) * sc),
              pack2<BF16>(__uint_as_float(v[8 * u + 2]) * sc, __uint_as_float(v[8 * u + 3]) * sc),
              pack2<BF16>(__uint_as_float(v[8 * u + 4]) * sc, __uint_as_float(v[8 * u + 5]) * sc),
              pack2<BF16>(__uint_as_float(v[8 * u + 6]) * sc, __uint_as_float(v[8 * u + 7]) * sc));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ dQ
// One CTA per 128-row query tile, walking the key tiles it can see.
// Tensor memory: S [0,128) | dP [128,256) (dS packed into it) | dQ [256, 256+D) |
// Q [384, 384+D/2) and dO [448, 448+D/2) packed 16-bit: the A operands of S = Q Kᵀ and
// dP = dO Vᵀ come from tensor memory, so per step the tensor core reads only K (twice)
// and V from shared memory.  S has one buffer, released as soon as the compute warps have
// loaded it, so S of the next step is computed while they exponentiate.
// Grid: x = query tile (fastest, sharing one head's K/V in L2; when causal the tile
// that sees the most key tiles first), y = head, z = batch or sequence.
template <int D, bool BF16>
__global__ void __launch_bounds__(384, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                     const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int BM = C::BM, BN = C::BN, VST = C::V_STAGES;
  constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DQ = 256, TM_QT = 384, TM_DOT = 448;
  constexpr int KST = C::K_STAGES;
  enum { B_QTM = 0, B_KFULL = 1, B_KEMPTY = B_KFULL + KST, B_VFULL = B_KEMPTY + KST,
         B_VEMPTY = B_VFULL + VST, B_SFULL = B_VEMPTY + VST, B_SEMPTY, B_DPFULL, B_DSFULL,
         B_DONE };
  static_assert(B_DONE < C::NBAR, "mbarrier slots");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::B_OFF_BAR + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + C::B_OFF_BAR + 8 * C::NBAR);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int h = blockIdx.y;
  const int bz = blockIdx.z;
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
    q_row0 = k_row0 = 0;
    Lq = Lk = p.N;
    bcoord = bz;
  }
  const int tile = p.reverse_tiles ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
  const int q0 = tile * BM;
  if (q0 >= Lq) return;
  const int diag = Lk - Lq;
  const int wl = p.win_left, wr = p.win_right;
  int j0, n_kv;  // key tiles j0 .. j0 + n_kv - 1
  key_tile_range(q0, min(q0 + BM - 1, Lq - 1), Lk, diag, wl, wr, BN, &j0, &n_kv);

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_QTM), 256);
    for (int s = 0; s < KST; ++s) {
      mbar_init(BAR(B_KFULL + s), 1);
      mbar_init(BAR(B_KEMPTY + s), 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(BAR(B_VFULL + s), 1);
      mbar_init(BAR(B_VEMPTY + s), 1);
    }
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_SEMPTY), 256);
    mbar_init(BAR(B_DPFULL), 1);
    mbar_init(BAR(B_DSFULL), 256);
    mbar_init(BAR(B_DONE), 1);
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

  if (warp == 0) {
    // ============================================================ loads
    if (lane == 0 && n_kv > 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      for (int j = 0; j < n_kv; ++j) {
        const int ks = j % KST, s = j % VST;
        mbar_wait(BAR(B_KEMPTY + ks), ((uint32_t)(j / KST) & 1u) ^ 1u, abort_flag, p.status);
        mbar_arrive_expect_tx(BAR(B_KFULL + ks), C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(&tmK, BAR(B_KFULL + ks), sbase + C::B_OFF_K + ks * C::TILE + c * C::CHUNK,
                      c * 64, h, k_row0 + (j0 + j) * BN, bcoord);
        mbar_wait(BAR(B_VEMPTY + s), ((uint32_t)(j / VST) & 1u) ^ 1u, abort_flag, p.status);
        mbar_arrive_expect_tx(BAR(B_VFULL + s), C::TILE);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(&tmV, BAR(B_VFULL + s), sbase + C::B_OFF_V + s * C::TILE + c * C::CHUNK,
                      c * 64, h, k_row0 + (j0 + j) * BN, bcoord);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t ID_S = idesc_f16_f32acc(BF16, 128, 128, false, false);   // S, dP
      constexpr uint32_t ID_DQ = idesc_f16_f32acc(BF16, 128, D, false, true);     // dQ
      // Descriptors built once; each MMA only adds a compile-time offset.
      const uint64_t dKk = sdesc_sw128(sbase + C::B_OFF_K, 16, 1024);         // K-major
      const uint64_t dKm = sdesc_sw128(sbase + C::B_OFF_K, C::CHUNK, 1024);   // MN-major
      const uint64_t dVk = sdesc_sw128(sbase + C::B_OFF_V, 16, 1024);
      // X = A Bᵀ with A (queries x d) packed in tensor memory and B = [keys][d] in shared
      // memory: K step kk covers d-elements 16kk.. = tensor-memory columns 8kk..
      auto issue_qt = [&](uint32_t dst, uint32_t a_tm, uint64_t db) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ts(tmem + dst, tmem + a_tm + 8u * kk,
                 sdesc_adv(db, (kk >> 2) * C::CHUNK + (kk & 3) * 32), ID_S, kk > 0 ? 1u : 0u);
      };
      auto issue_s = [&](int j) {  // S_j = Q K_jᵀ
        const int ks = j % KST;
        mbar_wait(BAR(B_KFULL + ks), (uint32_t)(j / KST) & 1u, abort_flag, p.status);
        tc_fence_after();
        issue_qt(TM_S, TM_QT, sdesc_adv(dKk, ks * C::TILE));
        mma_commit(BAR(B_SFULL));
      };
      auto issue_dp = [&](int j) {  // dP_j = dO V_jᵀ; V_j is free once it completes
        const int s = j % VST;
        mbar_wait(BAR(B_VFULL + s), (uint32_t)(j / VST) & 1u, abort_flag, p.status);
        tc_fence_after();
        issue_qt(TM_DP, TM_DOT, sdesc_adv(dVk, s * C::TILE));
        mma_commit(BAR(B_DPFULL));
        mma_commit(BAR(B_VEMPTY + s));
      };
      mbar_wait(BAR(B_QTM), 0, abort_flag, p.status);  // Q and dO are in tensor memory
      tc_fence_after();
      issue_s(0);
      issue_dp(0);
      for (int j = 0; j < n_kv; ++j) {
        const int ks = j % KST;
        // S_{j+1} as soon as the compute warps have loaded S_j
        if (j + 1 < n_kv) {
          mbar_wait(BAR(B_SEMPTY), (uint32_t)j & 1u, abort_flag, p.status);
          tc_fence_after();
          issue_s(j + 1);
        }
        // dQ += dS K_j  (A = dS in tensor memory; B = K_j as [d x keys], d-contiguous)
        mbar_wait(BAR(B_DSFULL), (uint32_t)j & 1u, abort_flag, p.status);
        tc_fence_after();
        const uint64_t kb = sdesc_adv(dKm, ks * C::TILE);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(tmem + TM_DQ, tmem + TM_DP + C::packed_col(kk), sdesc_adv(kb, kk * 2048), ID_DQ,
                 (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(BAR(B_KEMPTY + ks));
        // dP_{j+1} overwrites dS_j only after the product above that reads it (in-order)
        if (j + 1 < n_kv) issue_dp(j + 1);
      }
      mma_commit(BAR(B_DONE));
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ============================================================ compute: dS
    const int half = (warp - 4) >> 2;   // key columns 64*half .. 64*half+63
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within the tile
    const int i = q0 + r;               // query index within the sequence
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + TM_S + 64 * half;
    const uint32_t tDP = tmem + lane_off + TM_DP + 64 * half;
    const size_t grow = (p.cu_q != nullptr) ? ((size_t)(q_row0 + i) * p.H + h) * D
                                            : (((size_t)bcoord * p.N + i) * p.H + h) * D;
    {
      // this thread's row of Q (half 0) or dO (half 1) into tensor memory, packed 16-bit
      const uint4* src = reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint16_t*>(half == 0 ? p.q : p.dout) + grow);
      const uint32_t dst = tmem + lane_off + (half == 0 ? TM_QT : TM_DOT);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t w[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v = (i < Lq) ? src[c * 8 + u] : make_uint4(0u, 0u, 0u, 0u);
          w[4 * u] = v.x;
          w[4 * u + 1] = v.y;
          w[4 * u + 2] = v.z;
          w[4 * u + 3] = v.w;
        }
        tmem_st32(dst + 32u * c, w);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(B_QTM));
    }
    const float kLog2e = 1.4426950408889634f;
    float nl2 = -INFINITY, dd = 0.f;  // this row's -LSE·log2(e) and D
    if (i < Lq) {
      const size_t vi = (p.cu_q != nullptr) ? (size_t)h * p.total_q + q_row0 + i
                                            : ((size_t)bcoord * p.H + h) * p.N + i;
      nl2 = -p.lse[vi] * kLog2e;
      dd = p.dvec[vi];
    }
    const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
    const uint64_t nl22 = f2_pack(nl2, nl2);
    const uint64_t nd2 = f2_pack(-dd, -dd);
    for (int j = 0; j < n_kv; ++j) {
      const int kt = (j0 + j) * BN;       // first key of the tile
      const int k0 = kt + 64 * half;      // first key of this thread's columns
      const bool need_mask = (kt + BN > Lk) || (wr >= 0 && kt + BN - 1 > q0 + diag + wr) ||
                             (wl >= 0 && kt < q0 + BM - 1 + diag - wl);
      // allowed columns: lo <= c < lim
      const int lim = wr >= 0 ? min(Lk - k0, i + diag + wr - k0 + 1) : Lk - k0;
      const int lo = wl >= 0 ? i + diag - wl - k0 : 0;
      mbar_wait(BAR(B_SFULL), (uint32_t)j & 1u, abort_flag, p.status);
      tc_fence_after();
      uint32_t sv[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_wait_ld();
      reg_fence(sv);
      tc_fence_before();
      mbar_arrive(BAR(B_SEMPTY));  // S may be overwritten now
      float pv[64];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2 x = f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])),
                                          c2, nl22));
        pv[2 * e] = ex2_approx(x.x);
        pv[2 * e + 1] = ex2_approx(x.y);
      }
      if (need_mask) {
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (e >= lim || e < lo) pv[e] = 0.f;
      }
      mbar_wait(BAR(B_DPFULL), (uint32_t)j & 1u, abort_flag, p.status);
      tc_fence_after();
      uint32_t dv[64];
      tmem_ld32(tDP, *reinterpret_cast<uint32_t(*)[32]>(&dv[0]));
      tmem_ld32(tDP + 32, *reinterpret_cast<uint32_t(*)[32]>(&dv[32]));
      tmem_wait_ld();
      reg_fence(dv);
      uint32_t ds[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        // P is rounded to 16 bits first, as in the dK/dV pass and the forward P·V product
        const float2 pr = unpack2<BF16>(pack2<BF16>(pv[2 * e], pv[2 * e + 1]));
        const uint64_t t = f2_add(f2_pack(__uint_as_float(dv[2 * e]), __uint_as_float(dv[2 * e + 1])), nd2);
        const float2 d2 = f2_unpack(f2_mul(t, f2_pack(pr.x, pr.y)));
        ds[e] = pack2<BF16>(d2.x, d2.y);
      }
      tmem_st32(tDP, ds);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(B_DSFULL));
    }
    // ---------------------------------------------------------------- epilogue
    // dQ = scale · Σ dS K; half h stores columns [D/2 * h, D/2 * (h+1))
    if (n_kv > 0) {
      mbar_wait(BAR(B_DONE), 0, abort_flag, p.status);
      tc_fence_after();
    }
    uint16_t* orow = reinterpret_cast<uint16_t*>(p.dq) +
                     (p.cu_q != nullptr ? ((size_t)(q_row0 + i) * p.H + h) * D
                                        : (((size_t)bcoord * p.N + i) * p.H + h) * D);
    const float sc = p.scale;
#pragma unroll 1
    for (int q = half * (D / 64); q < (half + 1) * (D / 64); ++q) {
      uint32_t v[32];
      if (n_kv > 0) {
        tmem_ld32(tmem + lane_off + TM_DQ + q * 32, v);
        tmem_wait_ld();
        reg_fence(v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if (i < Lq) {
        uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          dst[u] = make_uint4(
              pack2<BF16>(__uint_as_float(v[8 * u]) * sc, __uint_as_float(v[8 * u + 1]) * sc),
              pack2<BF16>(__uint_as_float(v[8 * u + 2]) * sc, __uint_as_float(v[8 * u + 3]) * sc),
              pack2<BF16>(__uint_as_float(v[8 * u + 4]) * sc, __uint_as_float(v[8 * u + 5]) * sc),
              pack2<BF16>(__uint_as_float(v[8 * u + 6]) * sc, __uint_as_float(v[8 * u + 7]) * sc));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fattn
