// Single-pass backward of exact attention for sm_100a: one CTA per 128-key tile computes,
// for every query tile that can see its keys, the method's five products
//   Sᵀ = K Qᵀ,  dPᵀ = V dOᵀ,  dV += Pᵀ dO,  dK += dSᵀ Q,  dQ_i (+)= dS K
// and adds each dQ_i partial into an fp32 buffer shared by all key tiles (the "global
// gradients split into local updates" of page "Flash Attention V3：大模型训练加速与显存优化
// 技术解析" §3.2, with P recomputed from Q, K and the saved log-sum-exp as on the same page).
// With D_i = Σ_c dO_ic O_ic and P_ij = exp(scale q_i·k_j − LSE_i):
//   dS_ij = P_ij (dP_ij − D_i),  dQ_i = scale Σ_j dS_ij k_j,  dK_j = scale Σ_i dS_ij q_i,
//   dV_j = Σ_i P_ij dO_i
// (the chain rule applied to the "standard attention" of page "FlashAttention-2的核心设计原理").
//
// Kernels:
//   fa_bwd_pre_acc_kernel   D = rowsum(dO ∘ O) per (row, head), one warp each, and zeroes
//                           that row's fp32 dQ sums
//   fa_bwd_fused_kernel     the pass above
//   fa_bwd_dq_convert_kernel dQ = scale · sums, rounded to 16 bits
// launched in that order, each of the last two as a programmatic dependent of the one before
// (its CTAs may start early and wait for the preceding kernel only where they read its
// results).  CTAs of the pass run in groups of four (batch, head) pairs, tile-major inside a
// group (grouped_grid_item), each head's key tile 0 (the one with most query tiles when
// causal) first.
// dK and dV are written once per key tile (deterministic); the dQ sums are fp32 atomic adds
// whose order varies from run to run (the two-pass backward in bwd_kernel.cuh is the
// bitwise-reproducible alternative).
//
// CTA roles (16 warps): warp 0 loads (K, V once; Q through a 2-stage ring with the rows'
// LSE and D; dO one stage), warp 1 issues every tcgen05.mma from one thread, warps 4-11 are
// two compute warpgroups (thread = key row, one half of the 128 query columns each: Pᵀ into
// tensor memory, dSᵀ into shared memory), warps 12-15 drain each dQ partial from tensor
// memory into the fp32 sums (thread = query row) while the compute warps move on: 32 columns
// at a time go through two swizzled shared-memory staging tiles, which one thread hands to
// the TMA unit as reduce-adds into the sums; what does not fit in the tiles at once waits in
// registers, so tensor memory is released after one pass over the partial.
// Tensor memory: Sᵀ/Pᵀ [0,128) | dPᵀ [128,256) | dK [256,256+D) | dV [256+D,256+2D); the dQ
// partial (128 query lanes x D columns) takes the dPᵀ columns at D = 128 (free once the
// compute warps have loaded dPᵀ; the next dPᵀ waits for the drain) and columns [384,448) at
// D = 64.
// Shared memory: dS is stored [keys][queries] with the 128-byte swizzle, which is the
// K-major A operand of dK += dSᵀ Q and the MN-major A operand of dQ = dS K.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fattn_internal.h"
#include "sm100.cuh"

namespace fattn {

// ------------------------------------------------------------------ preprocess
// One warp per (token row, head): D = Σ_c dO·O into p.dvec (layout of lse) and the row's
// D fp32 dQ sums set to 0.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_pre_acc_kernel(const BwdParams p, long long rows_total) {
  // the fused pass is launched as a programmatic dependent of this kernel: its CTAs may start
  // (setup, K and V loads) while this one runs, and wait for its results where they use them
  grid_dependents_launch();
  constexpr int PER = D / 32;  // elements per lane
  const long long warps = (long long)gridDim.x * (blockDim.x / 32);
  const int lane = threadIdx.x & 31;
  for (long long w = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); w < rows_total * p.H;
       w += warps) {
    const long long row = w / p.H;
    const int h = (int)(w - row * p.H);
    const size_t base = (size_t)w * D + lane * PER;
    const uint16_t* o = reinterpret_cast<const uint16_t*>(p.o) + base;
    const uint16_t* g = reinterpret_cast<const uint16_t*>(p.dout) + base;
    float acc = 0.f;
    uint32_t av[PER / 2], bv[PER / 2];
    if constexpr (PER == 4) {
      const uint2 a = *reinterpret_cast<const uint2*>(o);
      const uint2 b = *reinterpret_cast<const uint2*>(g);
      av[0] = a.x; av[1] = a.y; bv[0] = b.x; bv[1] = b.y;
    } else {
      av[0] = *reinterpret_cast<const uint32_t*>(o);
      bv[0] = *reinterpret_cast<const uint32_t*>(g);
    }
#pragma unroll
    for (int e = 0; e < PER / 2; ++e) {
      const float2 fa = unpack2<BF16>(av[e]);
      const float2 fb = unpack2<BF16>(bv[e]);
      acc = fmaf(fa.x, fb.x, acc);
      acc = fmaf(fa.y, fb.y, acc);
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
    // zero the row's dQ sums ([rows, H, D], like dq): lane l clears columns 4l .. 4l+3
#pragma unroll
    for (int c = lane * 4; c < D; c += 128)
      *reinterpret_cast<float4*>(p.dq_acc + (size_t)w * D + c) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// ------------------------------------------------------------------ dQ conversion
// dQ = scale · sums, rounded to 16 bits; the sums and dq share the [rows, H, D] layout, so
// each thread converts 8 consecutive elements (two float4 reads, one 16-byte write).
template <bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_kernel(const BwdParams p, long long elems) {
  grid_dependency_wait();  // a programmatic dependent of the fused pass: its sums are complete
  const long long n8 = elems >> 3;  // D is a multiple of 8
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(p.dq_acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(p.dq_acc)[2 * i + 1];
    const float sc = p.scale;
    reinterpret_cast<uint4*>(p.dq)[i] =
        make_uint4(pack2<BF16>(a.x * sc, a.y * sc), pack2<BF16>(a.z * sc, a.w * sc),
                   pack2<BF16>(b.x * sc, b.y * sc), pack2<BF16>(b.z * sc, b.w * sc));
  }
}

// ------------------------------------------------------------------ fused pass
template <int D>
struct BwdFusedCfg {
  static constexpr int BM = 128;  // query rows per tile
  static constexpr int BN = 128;  // keys per tile
  static constexpr int KCH = D / 64;
  static constexpr int CHUNK = 128 * 128;  // one 64-column chunk of a 128-row tile
  static constexpr int TILE = 128 * D * 2;
  static constexpr int DS_TILE = 128 * 128 * 2;  // dSᵀ [keys][queries], 16-bit
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;             // 2 stages
#ifndef FATTN_BWD_DO_STAGES
#define FATTN_BWD_DO_STAGES 1
#endif
  static constexpr int DO_ST = FATTN_BWD_DO_STAGES;      // dO stages (1 or 2)
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;
  static constexpr int OFF_DS = OFF_DO + DO_ST * TILE;
  static constexpr int STG_TILE = 128 * 128;            // dQ staging: 128 rows x 32 fp32
  static constexpr int OFF_STG = OFF_DS + DS_TILE;       // 2 staging tiles
  static constexpr int OFF_VEC = OFF_STG + 2 * STG_TILE; // per Q stage: -lse*log2e [128], D [128]
  static constexpr int OFF_BAR = OFF_VEC + 2 * 2 * BM * 4;
  static constexpr int NBAR = 16;
  // The dynamic shared memory base is 1024-byte aligned on sm_100 (it follows the 1 KB the
  // driver reserves per CTA); the kernel checks that instead of reserving slack for it.
  static constexpr int SMEM = OFF_BAR + 8 * NBAR + 16;
  static_assert(SMEM <= 232448, "shared memory per CTA");
  static constexpr int THREADS = 512;
#ifndef FATTN_BWD_POLY_QUADS
#define FATTN_BWD_POLY_QUADS 4
#endif
  // of the 16 groups of 4 exponentials per thread and step, those taken by exp2_poly2
  static constexpr int kPolyQuads = FATTN_BWD_POLY_QUADS;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DK = 256, TM_DV = 256 + D;
  // the dQ partial: over dPᵀ at D = 128 (then the next dPᵀ waits for the drain)
  static constexpr uint32_t TM_DQ = D == 128 ? 128u : 384u;
  static constexpr bool DQ_ALIASES_DP = D == 128;
  __device__ static constexpr uint32_t packed_col(int kk) {
    return (uint32_t)(kk * 8 + (kk >= 4 ? 32 : 0));
  }
};

// PACKED: the packed varlen grid (packed_tile_lookup), in an instance of its own so that the
// lookup's code stays out of the other launches' kernels.
template <int D, bool BF16, bool PACKED = false>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                        const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDK,
                        const __grid_constant__ CUtensorMap tmDV, const BwdParams p) {
  using C = BwdFusedCfg<D>;
  constexpr int BM = C::BM, BN = C::BN;
  enum { B_KV = 0, B_QFULL = 1, B_QEMPTY = 3, B_DOFULL = 5, B_DOEMPTY = 7, B_SFULL = 9, B_DPFULL, B_PFULL,
         B_DSFULL, B_DQFULL, B_DQEMPTY, B_DONE };
  static_assert(B_DONE < C::NBAR, "mbarrier slots");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  if ((sbase & 1023u) != 0u) {  // the 128-byte swizzled tiles need 1024-byte atoms
    if (threadIdx.x == 0) atomicOr(p.status, kDevSmemAlign);
    return;
  }
  // the dQ conversion may be scheduled once every CTA of this grid has started (it waits for
  // this grid's completion before reading the sums)
  grid_dependents_launch();
  uint8_t* sgen = smem_raw;
  auto BAR = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + C::OFF_BAR + 8 * C::NBAR);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // grid: x = key tile, y = head, z = batch or sequence (a packed varlen grid: x = the key
  // tiles of all sequences, z = 1), launched in groups of heads that share L2 (their Q, dO
  // and dQ sums; see grouped_tile_order), key tile 0 (the one that sees the most query tiles
  // when causal) first
#ifndef FATTN_BWD_HEAD_GROUP
#define FATTN_BWD_HEAD_GROUP 4
#endif
  const GridItem item = grouped_tile_order(FATTN_BWD_HEAD_GROUP);
  const int h = item.h;
  int bz = item.bz;
  int ktile = item.tile;  // key tile within the batch or sequence
  int Lq, Lk, q_row0, k_row0, bcoord;
  if (p.cu_q != nullptr) {
    if constexpr (PACKED) {  // x numbers the key tiles of all segments, one after another
      if (blockIdx.x == 0 && blockIdx.y == 0)
        varlen_check_all(p.cu_q, p.cu_k, p.num_seqs, p.total_q, p.total_k, p.max_seqlen_q,
                         p.max_seqlen_k, p.status);
      if (!packed_tile_lookup(p.cu_k, p.num_seqs, p.total_k, item.tile, &bz, &ktile)) return;
    }
    if (!varlen_segment_ok(p.cu_q, p.cu_k, bz, p.total_q, p.total_k, p.max_seqlen_q,
                           p.max_seqlen_k, p.status))
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
  const int k0 = ktile * BN;
  if (k0 >= Lk) return;
  const int diag = Lk - Lq;
  const int wl = p.win_left, wr = p.win_right;
  int i_begin, n_q;  // query tiles i_begin .. i_begin + n_q - 1
  query_tile_range(k0, min(k0 + BN - 1, Lk - 1), Lq, diag, wl, wr, BM, &i_begin, &n_q);
  // Without a right bound every key tile starts at the same query tile: rotate the order per
  // key tile so that CTAs running together add into different dQ rows.
  const int rot = (wr < 0 && n_q > 0) ? ktile % n_q : 0;
  auto q_tile = [&](int it) { int t = it + rot; if (t >= n_q) t -= n_q; return i_begin + t; };
  // token row of query 0 of this sequence in the dQ sums
  const long long acc_row0 = (p.cu_q != nullptr) ? (long long)q_row0 : (long long)bcoord * p.N;

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_KV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(B_QFULL + s), 32);
      mbar_init(BAR(B_QEMPTY + s), 1);
    }
    for (int s = 0; s < C::DO_ST; ++s) {
      mbar_init(BAR(B_DOFULL + s), 1);
      mbar_init(BAR(B_DOEMPTY + s), 1);
    }
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_DPFULL), 1);
    mbar_init(BAR(B_PFULL), 256);
    mbar_init(BAR(B_DSFULL), 256);
    mbar_init(BAR(B_DQFULL), 1);
    mbar_init(BAR(B_DQEMPTY), 128);
    mbar_init(BAR(B_DONE), 1);
    *abort_flag = 0u;
    fence_barrier_init();
    // Thread 0 is the loads warp's lane: this key tile's K and V are requested right away,
    // so that their DRAM latency overlaps the tensor-memory allocation and the setup barrier.
    if (n_q > 0) {
      mbar_arrive_expect_tx(BAR(B_KV), 2 * C::TILE);
      for (int c = 0; c < C::KCH; ++c) {
        tma_load_4d(&tmK, BAR(B_KV), sbase + C::OFF_K + c * C::CHUNK, c * 64, h, k_row0 + k0,
                    bcoord);
        tma_load_4d(&tmV, BAR(B_KV), sbase + C::OFF_V + c * C::CHUNK, c * 64, h, k_row0 + k0,
                    bcoord);
      }
    }
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
      if (lane == 0) {  // K and V were requested during setup
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmDO);
      }
      grid_dependency_wait();  // D comes from the preceding preprocess launch
      for (int it = 0; it < n_q; ++it) {
        const int s = it & 1;
        const int q0 = q_tile(it) * BM;
        // -LSE·log2(e) and D of the 128 query rows (rows past the sequence: -inf, 0), read
        // before the stage is free so that their latency overlaps the wait
        float nl2[4], dd[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qg = q0 + lane * 4 + e;
          nl2[e] = -INFINITY;
          dd[e] = 0.f;
          if (qg < Lq) {
            const size_t vi = (p.cu_q != nullptr) ? (size_t)h * p.total_q + q_row0 + qg
                                                  : ((size_t)bcoord * p.H + h) * p.N + qg;
            nl2[e] = -p.lse[vi] * kLog2e;
            dd[e] = p.dvec[vi];
          }
        }
        mbar_wait(BAR(B_QEMPTY + s), ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag, p.status);
        if (lane == 0) {  // the Q tile first; every lane arrives once its vector entries are written
          mbar_expect_tx(BAR(B_QFULL + s), C::TILE);
          for (int c = 0; c < C::KCH; ++c)
            tma_load_4d(&tmQ, BAR(B_QFULL + s), sbase + C::OFF_Q + s * C::TILE + c * C::CHUNK,
                        c * 64, h, q_row0 + q0, bcoord);
        }
        float* vec = reinterpret_cast<float*>(sgen + C::OFF_VEC + s * 2 * BM * 4);
        *reinterpret_cast<float4*>(&vec[lane * 4]) = make_float4(nl2[0], nl2[1], nl2[2], nl2[3]);
        *reinterpret_cast<float4*>(&vec[BM + lane * 4]) = make_float4(dd[0], dd[1], dd[2], dd[3]);
        mbar_arrive(BAR(B_QFULL + s));
        if (lane == 0) {
          // a dO stage is free once the dV product of its previous step has read it
          const int ds_ = it % C::DO_ST;
          mbar_wait(BAR(B_DOEMPTY + ds_), ((uint32_t)(it / C::DO_ST) & 1u) ^ 1u, abort_flag,
                    p.status);
          mbar_arrive_expect_tx(BAR(B_DOFULL + ds_), C::TILE);
          for (int c = 0; c < C::KCH; ++c)
            tma_load_4d(&tmDO, BAR(B_DOFULL + ds_), sbase + C::OFF_DO + ds_ * C::TILE + c * C::CHUNK,
                        c * 64, h, q_row0 + q0, bcoord);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0 && n_q > 0) {
      constexpr uint32_t ID_ST = idesc_f16_f32acc(BF16, 128, 128, false, false);  // Sᵀ, dPᵀ
      constexpr uint32_t ID_DV = idesc_f16_f32acc(BF16, 128, D, false, true);     // dV (A in TMEM)
      constexpr uint32_t ID_DK = idesc_f16_f32acc(BF16, 128, D, false, true);     // dK: A K-major
      constexpr uint32_t ID_DQ = idesc_f16_f32acc(BF16, 128, D, true, true);      // dQ: A MN-major
      // Descriptors built once; each MMA only adds a compile-time offset.
      const uint64_t dK = sdesc_sw128(sbase + C::OFF_K, 16, 1024);              // K-major
      const uint64_t dKm = sdesc_sw128(sbase + C::OFF_K, C::CHUNK, 1024);       // MN-major
      const uint64_t dV = sdesc_sw128(sbase + C::OFF_V, 16, 1024);
      const uint64_t dQk = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);
      const uint64_t dQm = sdesc_sw128(sbase + C::OFF_Q, C::CHUNK, 1024);
      const uint64_t dDOk = sdesc_sw128(sbase + C::OFF_DO, 16, 1024);
      const uint64_t dDOm = sdesc_sw128(sbase + C::OFF_DO, C::CHUNK, 1024);
      const uint64_t dSk = sdesc_sw128(sbase + C::OFF_DS, 16, 1024);            // dSᵀ K-major
      const uint64_t dSm = sdesc_sw128(sbase + C::OFF_DS, C::CHUNK, 1024);      // dS MN-major
      // X = A Bᵀ with A = [keys][d] and B = [queries][d], both K-major
      auto issue_kt = [&](uint32_t dst, uint64_t da, uint64_t db) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          mma_ss(tmem + dst, sdesc_adv(da, off), sdesc_adv(db, off), ID_ST, kk > 0 ? 1u : 0u);
        }
      };
      auto wait_q = [&](int it) {
        mbar_wait(BAR(B_QFULL + (it & 1)), (uint32_t)(it >> 1) & 1u, abort_flag, p.status);
        tc_fence_after();
      };
      auto issue_dp = [&](int it) {
        mbar_wait(BAR(B_DOFULL + it % C::DO_ST), (uint32_t)(it / C::DO_ST) & 1u, abort_flag,
                  p.status);
        tc_fence_after();
        issue_kt(C::TM_DP, dV, sdesc_adv(dDOk, (it % C::DO_ST) * C::TILE));
        mma_commit(BAR(B_DPFULL));
      };
      mbar_wait(BAR(B_KV), 0, abort_flag, p.status);
      wait_q(0);
      issue_kt(C::TM_S, dK, dQk);
      mma_commit(BAR(B_SFULL));
      issue_dp(0);
      for (int it = 0; it < n_q; ++it) {
        const int s = it & 1;
        const uint32_t ph = (uint32_t)it & 1u;
        // dV += Pᵀ dO  (A = Pᵀ packed in tensor memory over Sᵀ; B = dO [queries][d], MN-major)
        mbar_wait(BAR(B_PFULL), ph, abort_flag, p.status);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          mma_ts(tmem + C::TM_DV, tmem + C::TM_S + C::packed_col(kk),
                 sdesc_adv(dDOm, (it % C::DO_ST) * C::TILE + kk * 2048),
                 ID_DV, (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(BAR(B_DOEMPTY + it % C::DO_ST));
        // dQ  = dS K   (A = dS [queries][keys], the dSᵀ tile read MN-major; B = K [keys][d]
        //              MN-major), first, so that its drain overlaps the next Sᵀ and the dK
        //              product
        // dK += dSᵀ Q  (A = dSᵀ [keys][queries] K-major; B = Q [queries][d] MN-major)
        mbar_wait(BAR(B_DSFULL), ph, abort_flag, p.status);
        tc_fence_after();
        if (C::DQ_ALIASES_DP == false && it > 0) {
          // the dQ columns of the previous step must have been drained
          mbar_wait(BAR(B_DQEMPTY), (uint32_t)(it - 1) & 1u, abort_flag, p.status);
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ss(tmem + C::TM_DQ, sdesc_adv(dSm, kk * 2048), sdesc_adv(dKm, kk * 2048), ID_DQ,
                 kk > 0 ? 1u : 0u);
        mma_commit(BAR(B_DQFULL));
        if (it + 1 < n_q) {  // Sᵀ of the next step over Pᵀ, between the dQ and dK products
          wait_q(it + 1);
          issue_kt(C::TM_S, dK, sdesc_adv(dQk, (it + 1 & 1) * C::TILE));
          mma_commit(BAR(B_SFULL));
        }
        const uint64_t qm = sdesc_adv(dQm, s * C::TILE);
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          mma_ss(tmem + C::TM_DK, sdesc_adv(dSk, (kk >> 2) * C::CHUNK + (kk & 3) * 32),
                 sdesc_adv(qm, kk * 2048), ID_DK, (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(BAR(B_QEMPTY + s));
        if (it + 1 < n_q) {
          if constexpr (C::DQ_ALIASES_DP) {
            // the next dPᵀ overwrites this dQ partial: wait until it has been drained
            mbar_wait(BAR(B_DQEMPTY), ph, abort_flag, p.status);
            tc_fence_after();
          }
          issue_dp(it + 1);
        }
      }
      mma_commit(BAR(B_DONE));
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 12) {
    // ============================================================ compute: Pᵀ, dSᵀ
    const int half = (warp - 4) >> 2;   // query columns 64*half .. 64*half+63
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row within the tile
    const int kg = k0 + r;
    const bool key_ok = kg < Lk;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S + 64 * half;
    const uint32_t tDP = tmem + lane_off + C::TM_DP + 64 * half;
    const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
    const int cbase = 64 * half;
    // this thread's 128-byte row of dSᵀ: chunk `half`, row r, 16-byte units swizzled by r % 8
    uint8_t* ds_row = sgen + C::OFF_DS + half * C::CHUNK + r * 128;
    for (int it = 0; it < n_q; ++it) {
      const int s = it & 1;
      const uint32_t ph = (uint32_t)it & 1u;
      const int q0 = q_tile(it) * BM;
      const float* vec = reinterpret_cast<const float*>(sgen + C::OFF_VEC + s * 2 * BM * 4);
      const bool need_mask = (k0 + BN > Lk) || (q0 + BM > Lq) ||
                             (wr >= 0 && k0 + BN - 1 > q0 + diag + wr) ||
                             (wl >= 0 && k0 < q0 + BM - 1 + diag - wl);
      const int qmin = wr >= 0 ? kg - diag - wr - q0 : -1;
      const int qend = wl >= 0 ? min(Lq - q0, kg - diag + wl - q0 + 1) : Lq - q0;
      mbar_wait(BAR(B_QFULL + s), (uint32_t)(it >> 1) & 1u, abort_flag, p.status);
      mbar_wait(BAR(B_SFULL), ph, abort_flag, p.status);
      tc_fence_after();
      uint32_t sv[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_wait_ld();
      reg_fence(sv);
      // p = 2^(s*c - LSE*log2e), masks applied afterwards on boundary tiles only
      const float4* nl4 = reinterpret_cast<const float4*>(&vec[cbase]);
      float pv[64];
#pragma unroll
      for (int e4 = 0; e4 < 16; ++e4) {
        const float4 nl = nl4[e4];
        const float2 x0 = f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[4 * e4]), __uint_as_float(sv[4 * e4 + 1])),
                                           c2, f2_pack(nl.x, nl.y)));
        const float2 x1 = f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[4 * e4 + 2]), __uint_as_float(sv[4 * e4 + 3])),
                                           c2, f2_pack(nl.z, nl.w)));
        if (e4 < C::kPolyQuads) {  // on the FMA pipe, beside the special-function unit
          const float2 y0 = exp2_poly2(x0.x, x0.y), y1 = exp2_poly2(x1.x, x1.y);
          pv[4 * e4] = y0.x;
          pv[4 * e4 + 1] = y0.y;
          pv[4 * e4 + 2] = y1.x;
          pv[4 * e4 + 3] = y1.y;
        } else {
          pv[4 * e4] = ex2_approx(x0.x);
          pv[4 * e4 + 1] = ex2_approx(x0.y);
          pv[4 * e4 + 2] = ex2_approx(x1.x);
          pv[4 * e4 + 3] = ex2_approx(x1.y);
        }
      }
      if (need_mask) {
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

      // dSᵀ = Pᵀ ∘ (dPᵀ − D) → 16-bit, into this thread's row of the shared dSᵀ tile.  The
      // tile is free: the previous step's dK and dQ products (its readers) completed before
      // this step's dPᵀ, which the wait below implies (tcgen05 products complete in order).
      mbar_wait(BAR(B_DPFULL), ph, abort_flag, p.status);
      tc_fence_after();
      uint32_t dv[64];
      tmem_ld32(tDP, *reinterpret_cast<uint32_t(*)[32]>(&dv[0]));
      tmem_ld32(tDP + 32, *reinterpret_cast<uint32_t(*)[32]>(&dv[32]));
      tmem_wait_ld();
      reg_fence(dv);
      const float4* d4 = reinterpret_cast<const float4*>(&vec[BM + cbase]);
#pragma unroll
      for (int u = 0; u < 8; ++u) {  // 16-byte unit u = queries cbase + 8u .. + 7
        uint32_t w[4];
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
          const int e4 = 2 * u + e2;
          const float4 dd = d4[e4];
          const float2 pa = unpack2<BF16>(pk[2 * e4]);
          const float2 pb = unpack2<BF16>(pk[2 * e4 + 1]);
          const float2 da = f2_unpack(f2_mul(f2_add(f2_pack(__uint_as_float(dv[4 * e4]), __uint_as_float(dv[4 * e4 + 1])),
                                                    f2_pack(-dd.x, -dd.y)),
                                             f2_pack(pa.x, pa.y)));
          const float2 db = f2_unpack(f2_mul(f2_add(f2_pack(__uint_as_float(dv[4 * e4 + 2]), __uint_as_float(dv[4 * e4 + 3])),
                                                    f2_pack(-dd.z, -dd.w)),
                                             f2_pack(pb.x, pb.y)));
          w[2 * e2] = pack2<BF16>(da.x, da.y);
          w[2 * e2 + 1] = pack2<BF16>(db.x, db.y);
        }
        *reinterpret_cast<uint4*>(ds_row + ((u ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();  // the tensor core reads the tile through the async proxy
      tc_fence_before();
      mbar_arrive(BAR(B_DSFULL));
    }
    // ---------------------------------------------------------------- epilogue
    // half 0 stores dV, half 1 stores dK = scale · Σ dSᵀ Q.  Whole key tiles (and every dense
    // tile: rows past N lie outside the tensor maps) leave through shared memory: each
    // thread writes its row into the V (dV) or K (dK) tile, free once the last product
    // completed, in the 128-byte swizzled layout, and one TMA store per 64-column chunk
    // writes whole rows.  The last, partial tile of a packed sequence is stored row by row,
    // so that it leaves the next sequence's rows alone.
    if (n_q > 0) {
      mbar_wait(BAR(B_DONE), 0, abort_flag, p.status);
      tc_fence_after();
    }
    uint16_t* orow = reinterpret_cast<uint16_t*>(half == 0 ? p.dv : p.dk) +
                     (p.cu_q != nullptr ? ((size_t)(k_row0 + kg) * p.H + h) * D
                                        : (((size_t)bcoord * p.N + kg) * p.H + h) * D);
    const float sc = half == 0 ? 1.f : p.scale;
    const uint32_t tsrc = tmem + lane_off + (half == 0 ? C::TM_DV : C::TM_DK);
    const bool via_tma = p.cu_q == nullptr || k0 + BN <= Lk;
    const int stage_off = half == 0 ? C::OFF_V : C::OFF_K;
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
      uint4 w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        w[u] = make_uint4(
            pack2<BF16>(__uint_as_float(v[8 * u]) * sc, __uint_as_float(v[8 * u + 1]) * sc),
            pack2<BF16>(__uint_as_float(v[8 * u + 2]) * sc, __uint_as_float(v[8 * u + 3]) * sc),
            pack2<BF16>(__uint_as_float(v[8 * u + 4]) * sc, __uint_as_float(v[8 * u + 5]) * sc),
            pack2<BF16>(__uint_as_float(v[8 * u + 6]) * sc, __uint_as_float(v[8 * u + 7]) * sc));
      if (via_tma) {
        // 16-byte unit u of row r of a chunk sits at r * 128 + ((u ^ (r % 8)) * 16)
        uint8_t* srow = sgen + stage_off + (q >> 1) * C::CHUNK + r * 128;
        const int u0 = (q & 1) * 4;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<uint4*>(srow + (((u0 + u) ^ (r & 7)) << 4)) = w[u];
      } else if (key_ok) {
        uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u) dst[u] = w[u];
      }
    }
    if (via_tma) {  // uniform over the CTA
      fence_proxy_async_smem();  // the rows above, visible to the TMA unit
      named_barrier_sync(2 + half, 128);
      if (quarter == 0 && lane == 0) {
        const CUtensorMap* map = half == 0 ? &tmDV : &tmDK;
        for (int c = 0; c < D / 64; ++c)
          tma_store_4d(map, sbase + stage_off + c * C::CHUNK, c * 64, h, k_row0 + k0, bcoord);
        bulk_commit_group();
        bulk_wait_group_read0();  // shared memory stays allocated until the TMA has read it
      }
    }
  } else if (warp >= 12) {
    // ============================================================ dQ drain
    // thread = query row (tensor-memory lane) of the partial; 32 columns at a time go through
    // two alternating shared-memory staging tiles (128-byte swizzle, the layout of the tensor
    // map's box) and one thread issues a TMA reduce-add per tile into the fp32 sums.  The
    // first two column groups are staged straight away (the tiles' previous reduce-adds, a
    // step ago, have read them by then), the rest is held in registers, so that the tensor
    // memory is released after one pass over it.  The TMA unit skips rows past the sums'
    // end; rows of this tile past the sequence carry zeros (their P is 0).
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const bool leader = threadIdx.x == 12 * 32;  // issues and waits for the reduce-adds
    constexpr int NG = D / 32;                   // 32-column groups
    constexpr int NS = 2;                        // staging tiles
#ifndef FATTN_BWD_DRAIN_FIRST
#define FATTN_BWD_DRAIN_FIRST 2
#endif
    // groups staged before the tensor memory is released; the others wait in registers
    constexpr int NF = FATTN_BWD_DRAIN_FIRST < NG ? FATTN_BWD_DRAIN_FIRST : NG;
    static_assert(NF >= 1 && NF <= NS, "drain staging");
    auto stage = [&](int c, const uint32_t (&g)[32]) {  // one group into tile c % NS
      uint8_t* row_ptr = sgen + C::OFF_STG + (c % NS) * C::STG_TILE + r * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<uint4*>(row_ptr + ((u ^ (r & 7)) << 4)) =
            make_uint4(g[4 * u], g[4 * u + 1], g[4 * u + 2], g[4 * u + 3]);
    };
    auto issue = [&](int c, int q0) {  // after the group's tile is complete
      fence_proxy_async_smem();
      named_barrier_sync(1, 128);
      if (leader) {
        tma_reduce_add_4d(&tmDQ, sbase + C::OFF_STG + (c % NS) * C::STG_TILE, 32 * c, h,
                          (int)(acc_row0 + q0), 0);
        bulk_commit_group();
      }
    };
    if (leader) tma_prefetch_desc(&tmDQ);
    grid_dependency_wait();  // the sums are zeroed by the preceding preprocess launch
    for (int it = 0; it < n_q; ++it) {
      const int q0 = q_tile(it) * BM;
      mbar_wait(BAR(B_DQFULL), (uint32_t)it & 1u, abort_flag, p.status);
      tc_fence_after();
      if (leader) bulk_wait_group_read0();  // the previous partial's tiles have been read
      named_barrier_sync(1, 128);
#pragma unroll
      for (int c = 0; c < NF; ++c) {  // staged straight away
        uint32_t g[32];
        tmem_ld32(tmem + lane_off + C::TM_DQ + 32 * c, g);
        tmem_wait_ld();
        reg_fence(g);
        stage(c, g);
      }
      uint32_t held[NG > NF ? NG - NF : 1][32];  // held in registers until a tile is free
      if constexpr (NG > NF) {
#pragma unroll
        for (int c = NF; c < NG; ++c) tmem_ld32(tmem + lane_off + C::TM_DQ + 32 * c, held[c - NF]);
        tmem_wait_ld();
#pragma unroll
        for (int c = NF; c < NG; ++c) reg_fence(held[c - NF]);
      }
      // the partial has been read: the next dPᵀ may overwrite its tensor-memory columns
      tc_fence_before();
      mbar_arrive(BAR(B_DQEMPTY));
#pragma unroll
      for (int c = 0; c < NF; ++c) issue(c, q0);
      if constexpr (NG > NF) {
#pragma unroll
        for (int c = NF; c < NG; ++c) {
          // tile c % NS: from the step's start it was free; reused, its reduce-add has read it
          if (c >= NS && leader) bulk_wait_group_read1();
          named_barrier_sync(1, 128);
          stage(c, held[c - NF]);
          issue(c, q0);
        }
      }
    }
    // The staging tiles must stay allocated until the TMA unit has read them.  Completion of
    // the reduce-adds themselves is not waited for here: the dQ conversion, a programmatic
    // dependent, waits for this grid's completion and the visibility of its memory operations.
    if (leader) bulk_wait_group_read0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fattn
