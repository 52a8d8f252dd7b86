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
// Kernels:
//   fa_bwd_pre_kernel   D = rowsum(dO ∘ O) (warp-shuffle reduction), dQ accumulator = 0
//   fa_bwd_kernel       one CTA per 128-key tile: loops over the 128-row query tiles
//                       that can see the tile; all five products on tcgen05
//   fa_bwd_dq_kernel    dQ = scale · accumulator, rounded to 16 bits
//
// Main-kernel roles: warp 0 loads (TMA for K, V once and Q_i, dO_i per step; plain
// loads for LSE_i, D_i), warp 1 issues tcgen05.mma, warps 2..5 ("compute") own one key
// row each (tensor-memory lane) and form Pᵀ and dSᵀ, warps 6..9 ("dq") drain the dQ
// tile from tensor memory into the fp32 accumulator with vector atomics.
// Tensor memory: Sᵀ (Pᵀ aliased as packed 16-bit) | dPᵀ (dQ_i aliased after dSᵀ is
// formed) | dK | dV.
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
      *reinterpret_cast<float4*>(p.dq_acc + base) = make_float4(0.f, 0.f, 0.f, 0.f);
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
      *reinterpret_cast<float2*>(p.dq_acc + base) = make_float2(0.f, 0.f);
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

// ------------------------------------------------------------------ dQ conversion
template <bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const float* __restrict__ acc,
                                                        uint16_t* __restrict__ dq, long long n8,
                                                        float scale) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += stride) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    uint4 r;
    r.x = pack2<BF16>(a.x * scale, a.y * scale);
    r.y = pack2<BF16>(a.z * scale, a.w * scale);
    r.z = pack2<BF16>(b.x * scale, b.y * scale);
    r.w = pack2<BF16>(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = r;
  }
}

// ------------------------------------------------------------------ main kernel
template <int D>
struct BwdCfg {
  static constexpr int BM = 128;  // query rows per step
  static constexpr int BN = 128;  // keys per CTA = tensor-memory lanes
  static constexpr int STAGES = 2;
  static constexpr int KCH = D / 64;
  static constexpr int CHUNK = 128 * 128;  // one 64-column chunk of a 128-row tile
  static constexpr int TILE = 128 * D * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;
  static constexpr int OFF_DO = OFF_Q + STAGES * TILE;
  static constexpr int OFF_DS = OFF_DO + STAGES * TILE;  // [key 128][query 128] 16-bit
  static constexpr int OFF_VEC = OFF_DS + 2 * CHUNK;      // per stage: lse2[128], D[128]
  static constexpr int OFF_BAR = OFF_VEC + STAGES * 2 * BM * 4;
  static constexpr int B_KV = 0;
  static constexpr int B_QFULL = 1;
  static constexpr int B_QEMPTY = B_QFULL + STAGES;
  static constexpr int B_SFULL = B_QEMPTY + STAGES;
  static constexpr int B_DPFULL = B_SFULL + 1;
  static constexpr int B_PFULL = B_DPFULL + 1;
  static constexpr int B_DSFULL = B_PFULL + 1;
  static constexpr int B_DSEMPTY = B_DSFULL + 1;
  static constexpr int B_DQFULL = B_DSEMPTY + 1;
  static constexpr int B_DQEMPTY = B_DQFULL + 1;
  static constexpr int B_DONE = B_DQEMPTY + 1;
  static constexpr int NBAR = B_DONE + 1;
  static constexpr int USED = OFF_BAR + 8 * NBAR + 16;
  static constexpr int SMEM_MAX = 232448;  // opt-in limit per CTA on sm_100
  static constexpr int SLACK = (USED + 1024 <= SMEM_MAX) ? 1024 : (SMEM_MAX - USED) & ~15;
  static constexpr int SMEM_BYTES = USED + SLACK;
  static constexpr int THREADS = 320;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DK = 256, TM_DV = 256 + D;
};

template <int D, bool BF16>
__global__ void __launch_bounds__(320, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int BM = C::BM, BN = C::BN, ST = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  if (pad > (uint32_t)C::SLACK) {  // cannot place 1024-byte aligned tiles: report, do nothing
    if (threadIdx.x == 0) atomicOr(p.status, kDevSmemAlign);
    return;
  }
  const uint32_t sbase = raw + pad;
  uint8_t* sgen = smem_raw + pad;
  auto BAR = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sgen + C::OFF_BAR + 8 * C::NBAR);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---------------------------------------------------------------- work item
  const int h = blockIdx.y;
  int Lq, Lk, q_row0, k_row0, bcoord;
  if (p.cu_q != nullptr) {
    const int s = blockIdx.z;
    q_row0 = p.cu_q[s];
    Lq = p.cu_q[s + 1] - q_row0;
    k_row0 = p.cu_k[s];
    Lk = p.cu_k[s + 1] - k_row0;
    bcoord = 0;
  } else {
    q_row0 = k_row0 = 0;
    Lq = Lk = p.N;
    bcoord = blockIdx.z;
  }
  const int k0 = blockIdx.x * BN;
  if (k0 >= Lk) return;
  const int diag = Lk - Lq;
  const int q_tiles = (Lq + BM - 1) / BM;
  int i_begin = 0;
  if (p.causal) {
    const int first_q = k0 - diag;  // first query row that may see key k0
    i_begin = first_q <= 0 ? 0 : first_q / BM;
  }
  const int n_q = q_tiles > i_begin ? q_tiles - i_begin : 0;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    mbar_init(BAR(C::B_KV), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(BAR(C::B_QFULL + s), 32);
      mbar_init(BAR(C::B_QEMPTY + s), 1);
    }
    mbar_init(BAR(C::B_SFULL), 1);
    mbar_init(BAR(C::B_DPFULL), 1);
    mbar_init(BAR(C::B_PFULL), 128);
    mbar_init(BAR(C::B_DSFULL), 128);
    mbar_init(BAR(C::B_DSEMPTY), 1);
    mbar_init(BAR(C::B_DQFULL), 1);
    mbar_init(BAR(C::B_DQEMPTY), 128);
    mbar_init(BAR(C::B_DONE), 1);
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
        mbar_arrive_expect_tx(BAR(C::B_KV), 2 * C::TILE);
        for (int c = 0; c < C::KCH; ++c) {
          tma_load_4d(&tmK, BAR(C::B_KV), sbase + C::OFF_K + c * C::CHUNK, c * 64, h, k_row0 + k0,
                      bcoord);
          tma_load_4d(&tmV, BAR(C::B_KV), sbase + C::OFF_V + c * C::CHUNK, c * 64, h, k_row0 + k0,
                      bcoord);
        }
      }
      for (int it = 0; it < n_q; ++it) {
        const int s = it % ST;
        const int q0 = (i_begin + it) * BM;
        mbar_wait(BAR(C::B_QEMPTY + s), ((uint32_t)(it / ST) & 1u) ^ 1u, abort_flag, p.status);
        // LSE (as log2 units) and D for the 128 query rows of this step; rows past the
        // sequence get LSE = +inf (P = 0) and D = 0.
        float* vec = reinterpret_cast<float*>(sgen + C::OFF_VEC + s * 2 * BM * 4);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qc = lane * 4 + e;
          const int qg = q0 + qc;
          float l2 = INFINITY, dd = 0.f;
          if (qg < Lq) {
            size_t vi = (p.cu_q != nullptr) ? (size_t)h * p.total_q + q_row0 + qg
                                            : ((size_t)bcoord * p.H + h) * p.N + qg;
            l2 = p.lse[vi] * kLog2e;
            dd = p.dvec[vi];
          }
          vec[qc] = l2;
          vec[BM + qc] = dd;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(BAR(C::B_QFULL + s), 2 * C::TILE);
          for (int c = 0; c < C::KCH; ++c) {
            tma_load_4d(&tmQ, BAR(C::B_QFULL + s), sbase + C::OFF_Q + s * C::TILE + c * C::CHUNK,
                        c * 64, h, q_row0 + q0, bcoord);
            tma_load_4d(&tmDO, BAR(C::B_QFULL + s), sbase + C::OFF_DO + s * C::TILE + c * C::CHUNK,
                        c * 64, h, q_row0 + q0, bcoord);
          }
        } else {
          mbar_arrive(BAR(C::B_QFULL + s));
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0 && n_q > 0) {
      constexpr uint32_t ID_SS_KK = idesc_f16_f32acc(BF16, 128, 128, false, false);  // Sᵀ, dPᵀ
      constexpr uint32_t ID_KMN = idesc_f16_f32acc(BF16, 128, D, false, true);       // dV, dK
      constexpr uint32_t ID_MNMN = idesc_f16_f32acc(BF16, 128, D, true, true);       // dQ
      const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sDS = sbase + C::OFF_DS;
      mbar_wait(BAR(C::B_KV), 0, abort_flag, p.status);
      for (int it = 0; it < n_q; ++it) {
        const int s = it % ST;
        const uint32_t ph = (uint32_t)it & 1u;
        const uint32_t sQ = sbase + C::OFF_Q + s * C::TILE;
        const uint32_t sDO = sbase + C::OFF_DO + s * C::TILE;
        mbar_wait(BAR(C::B_QFULL + s), (uint32_t)(it / ST) & 1u, abort_flag, p.status);
        tc_fence_after();
        // Sᵀ = K Qᵀ   (M = keys, N = queries, K = d; both operands K-major)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          mma_ss(tmem + C::TM_S, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(sQ + off, 16, 1024),
                 ID_SS_KK, kk > 0 ? 1u : 0u);
        }
        mma_commit(BAR(C::B_SFULL));
        // dPᵀ = V dOᵀ, written where dQ of the previous step lived: wait until drained.
        if (it > 0) mbar_wait(BAR(C::B_DQEMPTY), ph ^ 1u, abort_flag, p.status);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          mma_ss(tmem + C::TM_DP, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(sDO + off, 16, 1024),
                 ID_SS_KK, kk > 0 ? 1u : 0u);
        }
        mma_commit(BAR(C::B_DPFULL));
        // dV += Pᵀ dO   (A = Pᵀ in tensor memory; B = dO as [d x queries], d-contiguous)
        mbar_wait(BAR(C::B_PFULL), ph, abort_flag, p.status);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          mma_ts(tmem + C::TM_DV, tmem + C::TM_S + kk * 8,
                 sdesc_sw128(sDO + kk * 2048, C::CHUNK, 1024), ID_KMN, (it > 0 || kk > 0) ? 1u : 0u);
        // dK += dSᵀ Q   (A = dSᵀ [keys x queries] K-major; B = Q as [d x queries])
        mbar_wait(BAR(C::B_DSFULL), ph, abort_flag, p.status);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint32_t offa = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          mma_ss(tmem + C::TM_DK, sdesc_sw128(sDS + offa, 16, 1024),
                 sdesc_sw128(sQ + kk * 2048, C::CHUNK, 1024), ID_KMN, (it > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(BAR(C::B_QEMPTY + s));
        // dQ_i = dS K   (M = queries: A = dS read from the [key][query] buffer, query-
        // contiguous = MN-major; B = K as [d x keys], d-contiguous), into dPᵀ's columns.
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ss(tmem + C::TM_DP, sdesc_sw128(sDS + kk * 2048, C::CHUNK, 1024),
                 sdesc_sw128(sK + kk * 2048, C::CHUNK, 1024), ID_MNMN, kk > 0 ? 1u : 0u);
        mma_commit(BAR(C::B_DSEMPTY));
        mma_commit(BAR(C::B_DQFULL));
      }
      mma_commit(BAR(C::B_DONE));
    }
    __syncwarp();
  } else if (warp < 6) {
    // ============================================================ compute: Pᵀ, dSᵀ
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row within the tile
    const int kg = k0 + r;              // key index within the sequence
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S;
    const uint32_t tDP = tmem + lane_off + C::TM_DP;
    const float c = p.scale_log2;
    uint8_t* ds_row = sgen + C::OFF_DS + r * 128;
    for (int it = 0; it < n_q; ++it) {
      const int s = it % ST;
      const uint32_t ph = (uint32_t)it & 1u;
      const int q0 = (i_begin + it) * BM;
      const float* vec = reinterpret_cast<const float*>(sgen + C::OFF_VEC + s * 2 * BM * 4);
      const bool need_mask =
          (k0 + BN > Lk) || (q0 + BM > Lq) || (p.causal && (k0 + BN - 1 > q0 + diag));
      // Allowed queries for this key: q >= kg - diag (causal) and q < Lq.
      const int qmin = p.causal ? kg - diag - q0 : -1;  // column index bound
      const bool key_ok = kg < Lk;
      mbar_wait(BAR(C::B_QFULL + s), (uint32_t)(it / ST) & 1u, abort_flag, p.status);
      mbar_wait(BAR(C::B_SFULL), ph, abort_flag, p.status);
      tc_fence_after();
      uint32_t pk[64];  // Pᵀ row as packed 16-bit pairs
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t sv[32];
        tmem_ld32(tS + q * 32, sv);
        tmem_wait_ld();
        reg_fence(sv);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c0 = q * 32 + 2 * e;
          float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * e]), c, -vec[c0]));
          float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * e + 1]), c, -vec[c0 + 1]));
          if (need_mask) {
            if (!key_ok || c0 < qmin || q0 + c0 >= Lq) p0 = 0.f;
            if (!key_ok || c0 + 1 < qmin || q0 + c0 + 1 >= Lq) p1 = 0.f;
          }
          pk[q * 16 + e] = pack2<BF16>(p0, p1);
        }
        tmem_st16(tS + q * 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[q * 16]));
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(C::B_PFULL));

      // dSᵀ = Pᵀ ∘ (dPᵀ − D) into shared memory, 128-byte swizzled [key][query].
      mbar_wait(BAR(C::B_DPFULL), ph, abort_flag, p.status);
      if (it > 0) mbar_wait(BAR(C::B_DSEMPTY), ph ^ 1u, abort_flag, p.status);
      tc_fence_after();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t dv[32];
        tmem_ld32(tDP + q * 32, dv);
        tmem_wait_ld();
        reg_fence(dv);
        uint32_t o[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c0 = q * 32 + 2 * e;
          float2 pf;
          if constexpr (BF16)
            pf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[q * 16 + e]));
          else
            pf = __half22float2(*reinterpret_cast<const __half2*>(&pk[q * 16 + e]));
          const float d0 = pf.x * (__uint_as_float(dv[2 * e]) - vec[BM + c0]);
          const float d1 = pf.y * (__uint_as_float(dv[2 * e + 1]) - vec[BM + c0 + 1]);
          o[e] = pack2<BF16>(d0, d1);
        }
        // columns q*32 .. q*32+31 = chunk (q/2), 16-byte units (q%2)*4 .. +3
        const int chunk = q >> 1;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int unit = (q & 1) * 4 + u;
          uint4* dst = reinterpret_cast<uint4*>(ds_row + chunk * C::CHUNK + ((unit ^ (r & 7)) << 4));
          *dst = make_uint4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(BAR(C::B_DSFULL));
    }
    // ---------------------------------------------------------------- dV epilogue
    if (n_q > 0) {
      mbar_wait(BAR(C::B_DONE), 0, abort_flag, p.status);
      tc_fence_after();
    }
    uint16_t* dvrow = reinterpret_cast<uint16_t*>(p.dv) +
                      (p.cu_q != nullptr ? ((size_t)(k_row0 + kg) * p.H + h) * D
                                         : (((size_t)bcoord * p.N + kg) * p.H + h) * D);
#pragma unroll 1
    for (int q = 0; q < D / 32; ++q) {
      uint32_t v[32];
      if (n_q > 0) {
        tmem_ld32(tmem + lane_off + C::TM_DV + q * 32, v);
        tmem_wait_ld();
        reg_fence(v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if (kg < Lk) {
        uint4* dst = reinterpret_cast<uint4*>(dvrow + q * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          dst[u] = make_uint4(pack2<BF16>(__uint_as_float(v[8 * u]), __uint_as_float(v[8 * u + 1])),
                              pack2<BF16>(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3])),
                              pack2<BF16>(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5])),
                              pack2<BF16>(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7])));
      }
    }
  } else {
    // ============================================================ dq: drain dQ_i, dK epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within the step (dQ) / key row (dK)
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tDQ = tmem + lane_off + C::TM_DP;
    for (int it = 0; it < n_q; ++it) {
      const uint32_t ph = (uint32_t)it & 1u;
      const int qg = (i_begin + it) * BM + r;
      mbar_wait(BAR(C::B_DQFULL), ph, abort_flag, p.status);
      tc_fence_after();
      float* dst = p.dq_acc + (p.cu_q != nullptr ? ((size_t)(q_row0 + qg) * p.H + h) * D
                                                 : (((size_t)bcoord * p.N + qg) * p.H + h) * D);
#pragma unroll 1
      for (int q = 0; q < D / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(tDQ + q * 32, v);
        tmem_wait_ld();
        reg_fence(v);
        if (qg < Lq) {
#pragma unroll
          for (int u = 0; u < 8; ++u)
            atomicAdd(reinterpret_cast<float4*>(dst + q * 32) + u,
                      make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]),
                                  __uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3])));
        }
      }
      tc_fence_before();
      mbar_arrive(BAR(C::B_DQEMPTY));
    }
    // dK = scale · (Σ dSᵀ Q)
    if (n_q > 0) {
      mbar_wait(BAR(C::B_DONE), 0, abort_flag, p.status);
      tc_fence_after();
    }
    const int kg = k0 + r;
    uint16_t* dkrow = reinterpret_cast<uint16_t*>(p.dk) +
                      (p.cu_q != nullptr ? ((size_t)(k_row0 + kg) * p.H + h) * D
                                         : (((size_t)bcoord * p.N + kg) * p.H + h) * D);
    const float sc = p.scale;
#pragma unroll 1
    for (int q = 0; q < D / 32; ++q) {
      uint32_t v[32];
      if (n_q > 0) {
        tmem_ld32(tmem + lane_off + C::TM_DK + q * 32, v);
        tmem_wait_ld();
        reg_fence(v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if (kg < Lk) {
        uint4* dst = reinterpret_cast<uint4*>(dkrow + q * 32);
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

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fattn
