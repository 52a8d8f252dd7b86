// KV-cache decode for sm_100a: a few new query tokens per sequence attend to the keys and
// values that sequence has cached, in a contiguous cache [B, capacity, H, d] or a paged
// cache [num_pages, page_size, H, d] addressed through a block table.
//
// Method (what is computed): the same exact softmax attention as the forward kernel, with
// the running maximum and rescaled running sum of the page "FlashAttention实战：如何在
// A100上实现3倍加速的Transformer训练" §3.1 applied twice: across the key tiles a CTA
// streams, and across the CTAs ("splits") that share one sequence's cache, whose partial
// results are merged by the same rule in log-sum-exp form.  KV caches for incremental
// decoding and paged KV caches are features the page "FlashAttention技术深度解析"
// (pwwt.cn/news/595117) lists without an interface; the new tokens are read as the last
// Nq positions of the cache (bottom-right alignment, as for causal masking).
//
// How it maps to B200.  Each cached key and value is read once and used for Nq·d
// multiply-adds, so the kernel is bound by HBM bandwidth, not by the tensor cores: the
// arithmetic runs on the CUDA cores and the design goal is to keep enough bytes in
// flight.
//   * grid (splits, H, B): a CTA takes one contiguous range of keys (a split, a multiple
//     of 128 keys) of one (sequence, head), so that short batches still cover all SMs;
//   * the last warp streams 128-key K and V tiles by TMA (128-byte swizzle) through a ring of
//     STAGES stages (192 KB of shared memory in flight per SM);
//   * compute warps in groups of four (two groups when Nq <= 4, so each SM
//     sub-partition has two compute warps to hide latency; group g takes tiles g, g + G,
//     ... with its own softmax state, merged at the end).  Scores: thread t of a group
//     owns key t of the tile and forms its dot
//     product with every query row (query rows in shared memory as fp32, read as
//     broadcasts; several independent partial sums per row so the FMAs do not wait on
//     each other).  Online softmax: the tile maximum of each row by warp shuffles and an
//     exchange of the four warps' maxima through shared memory; every thread then holds
//     the same running maximum, exponentiates its own key's scores and keeps its own
//     partial row sum (summed once at the end).  P·V: warp w takes keys 32w..32w+31 of
//     the tile, lane l the columns d/32·l ..; the four warps' partial outputs of the same
//     rows are added once at the end;
//   * one split: the CTA writes O and LSE; several: each writes its normalised partial O
//     (fp32) and log2-domain LSE to the caller's workspace and fa_decode_combine_kernel
//     merges them, O = Σ_s 2^(LSE_s − LSE) O_s with LSE = log2 Σ_s 2^LSE_s.
// Keys past a sequence's length are never multiplied into O (cache rows there may hold
// anything), and a paged tile loads only the pages that hold the sequence's keys.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fattn_internal.h"
#include "sm100.cuh"

namespace fattn {

template <int D, int NQ>
struct DecCfg {
  static constexpr int BN = 128;                   // keys per tile
  static constexpr int STAGES = (D == 128) ? 3 : 6;
  static constexpr int KCH = D / 64;               // 64-column (128-byte) chunks per row
  static constexpr int CHUNK = 128 * 128;          // one chunk of a 128-row tile
  static constexpr int TILE = 128 * D * 2;         // a K or a V tile
  static constexpr int CPL = D / 32;               // output columns per lane in P·V
  // consumer groups of four warps; group g takes tiles g, g + G, ...  Two groups give
  // each SM sub-partition two compute warps; sixteen query rows need the room for one.
  static constexpr int G = NQ <= 4 ? 2 : 1;
  static constexpr int OFF_Q = 2 * STAGES * TILE;  // stage s: K at 2s·TILE, V at (2s+1)·TILE
  static constexpr int OFF_S = OFF_Q + NQ * D * 4;          // fp32 [G][2][NQ][BN]: P
  static constexpr int OFF_WM = OFF_S + G * 2 * NQ * BN * 4;  // fp32 [G][2][4][NQ]: warp maxima
  static constexpr int OFF_L = OFF_WM + G * 2 * 4 * NQ * 4;   // fp32 [G][4][NQ]: warp sums
  static constexpr int OFF_M = OFF_L + G * 4 * NQ * 4;        // fp32 [G][NQ]: group maxima
  static constexpr int OFF_BAR = (OFF_M + G * NQ * 4 + 7) / 8 * 8;
  static constexpr int NBAR = 3 * STAGES;
  static constexpr int SMEM_BYTES = OFF_BAR + 8 * NBAR + 16 + 1024;  // + alignment slack
  static constexpr int THREADS = 128 * G + 32;  // compute warps, then one load warp
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(G * 4 * NQ * D * 4 <= 2 * STAGES * TILE, "final reduction fits in the ring");
};

template <bool BF16>
__device__ __forceinline__ float half_to_f32(uint16_t v) {
  if constexpr (BF16) {
    return __uint_as_float((uint32_t)v << 16);
  } else {
    return __half2float(__ushort_as_half(v));
  }
}

// NQ: compile-time bound on the query rows (p.Nq <= NQ); rows past p.Nq are skipped.
template <int D, bool BF16, bool PAGED, int NQ>
__global__ void __launch_bounds__(DecCfg<D, NQ>::THREADS, 1)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const DecParams p) {
  using C = DecCfg<D, NQ>;
  constexpr int BN = C::BN, ST = C::STAGES, CPL = C::CPL, G = C::G;
  constexpr int NCOMP = 128 * G;  // compute threads
  enum { B_KFULL = 0, B_VFULL = ST, B_EMPTY = 2 * ST };
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  auto BAR = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * (uint32_t)i; };
  volatile uint32_t* abort_flag =
      reinterpret_cast<volatile uint32_t*>(sgen + C::OFF_BAR + 8 * C::NBAR);
  float* qs = reinterpret_cast<float*>(sgen + C::OFF_Q);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int Nq = p.Nq;
  int L = p.seqlens[b];
  if (L < 0 || L > p.max_len) {  // a length the caller's bounds do not cover: report, clamp
    if (tid == 0) atomicOr(p.status, kDevBadCache);
    L = L < 0 ? 0 : p.max_len;
  }
  const int wl = p.win_left, wr = p.win_right;
  // keys any query row may see: [lo_all, L) (the last row's upper bound is >= L - 1)
  const int lo_all = wl >= 0 ? max(0, L - Nq - wl) : 0;
  const int k_first = max(split * p.chunk, lo_all) / BN * BN;
  const int k_end = min(L, (split + 1) * p.chunk);
  const int n_tiles = k_end > k_first ? (k_end - k_first + BN - 1) / BN : 0;

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(BAR(B_KFULL + s), 1);
      mbar_init(BAR(B_VFULL + s), 1);
      mbar_init(BAR(B_EMPTY + s), 4);  // one arrival per warp of the consuming group
    }
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (tid < NCOMP) {  // query rows as fp32
    const uint16_t* qg = reinterpret_cast<const uint16_t*>(p.q);
    for (int e = tid; e < Nq * D; e += NCOMP) {
      const int r = e / D, c = e - r * D;
      qs[r * D + c] = half_to_f32<BF16>(qg[((size_t)(b * Nq + r) * p.H + h) * D + c]);
    }
  }
  __syncthreads();

  if (warp == 4 * G) {
    // ============================================================ TMA producer
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t % ST;
        mbar_wait(BAR(B_EMPTY + s), ((uint32_t)(t / ST) & 1u) ^ 1u, abort_flag, p.status);
        const int k0 = k_first + t * BN;
        const uint32_t dK = sbase + (uint32_t)(2 * s) * C::TILE, dV = dK + C::TILE;
        if constexpr (!PAGED) {
          mbar_arrive_expect_tx(BAR(B_KFULL + s), C::TILE);
          for (int c = 0; c < C::KCH; ++c)
            tma_load_4d(&tmK, BAR(B_KFULL + s), dK + c * C::CHUNK, c * 64, h, k0, b);
          mbar_arrive_expect_tx(BAR(B_VFULL + s), C::TILE);
          for (int c = 0; c < C::KCH; ++c)
            tma_load_4d(&tmV, BAR(B_VFULL + s), dV + c * C::CHUNK, c * 64, h, k0, b);
        } else {
          // boxes of min(page_size, 128) rows; only those holding keys below L are loaded
          const int rows = min(p.page_size, BN);
          const int nload = min(BN / rows, (L - k0 + rows - 1) / rows);
          const uint32_t bytes = (uint32_t)(nload * rows * 128 * C::KCH);
          mbar_arrive_expect_tx(BAR(B_KFULL + s), bytes);
          mbar_arrive_expect_tx(BAR(B_VFULL + s), bytes);
          for (int i = 0; i < nload; ++i) {
            const int key = k0 + i * rows;
            const int page = p.block_table[(size_t)b * p.max_blocks + key / p.page_size];
            // an out-of-range page reads as zeros (TMA bounds) and is reported
            if (page < 0 || page >= p.num_pages) atomicOr(p.status, kDevBadCache);
            const int row = key % p.page_size;
            const uint32_t off = (uint32_t)(i * rows * 128);
            for (int c = 0; c < C::KCH; ++c) {
              tma_load_4d(&tmK, BAR(B_KFULL + s), dK + c * C::CHUNK + off, c * 64, h, row, page);
              tma_load_4d(&tmV, BAR(B_VFULL + s), dV + c * C::CHUNK + off, c * 64, h, row, page);
            }
          }
        }
      }
    }
    __syncwarp();
    return;
  }

  // ============================================================== compute groups
  // Group g (warps 4g..4g+3) takes tiles g, g + G, ...  Within a group every thread keeps
  // the running maximum m of every query row (identical in all its threads) and a partial
  // row sum l over the keys it owned; O partials per warp.  Groups merge at the end.
  const int g = warp >> 2, gw = warp & 3;  // group, warp within the group
  const int gt = tid & 127;                // thread within the group = key of the tile
  float* S = reinterpret_cast<float*>(sgen + C::OFF_S) + g * 2 * NQ * BN;
  float* WM = reinterpret_cast<float*>(sgen + C::OFF_WM) + g * 2 * 4 * NQ;
  float* LW = reinterpret_cast<float*>(sgen + C::OFF_L) + g * 4 * NQ;
  float* MG = reinterpret_cast<float*>(sgen + C::OFF_M);
  const uint32_t gbar = 1u + (uint32_t)g;  // named barrier of this group
  float m_run[NQ], l_run[NQ];
#pragma unroll
  for (int r = 0; r < NQ; ++r) {
    m_run[r] = -INFINITY;
    l_run[r] = 0.f;
  }
  float o[NQ][CPL];
#pragma unroll
  for (int r = 0; r < NQ; ++r)
#pragma unroll
    for (int e = 0; e < CPL; ++e) o[r][e] = 0.f;
  const float c = p.scale_log2;
  // independent partial dot products per row (breaks the FMA dependency chain)
  constexpr int NACC = NQ == 1 ? 8 : (NQ <= 4 ? 4 : 2);
  // up to four query rows: the score and P·V multiply-adds issue two lanes per instruction
  // (fma.rn.f32x2); sixteen rows keep the scalar form, which fits the registers
  constexpr bool PAIRED = NQ > 1 && NQ <= 4;
  // this lane's P·V columns: chunk, 16-byte segment and byte offset inside it
  const int col0 = lane * CPL;
  const int vchunk = col0 >> 6, vseg = (col0 & 63) >> 3, vbyte = (col0 & 7) * 2;

  for (int t = g, u = 0; t < n_tiles; t += G, ++u) {
    const int s = t % ST;
    const uint32_t ph = (uint32_t)(t / ST) & 1u;
    const int buf = u & 1;
    const int k0 = k_first + t * BN;
    const uint8_t* Ks = sgen + (2 * s) * C::TILE;
    const uint8_t* Vs = Ks + C::TILE;
    float* Sb = S + buf * NQ * BN;
    float* WMb = WM + buf * 4 * NQ;

    // ---- scores x = c · q_r·k_j (thread = key j), masked keys -inf
    mbar_wait(BAR(B_KFULL + s), ph, abort_flag, p.status);
    const int j = k0 + gt;
    float x[NQ];
    {
      float acc[NQ][NACC];
#pragma unroll
      for (int r = 0; r < NQ; ++r)
#pragma unroll
        for (int a = 0; a < NACC; ++a) acc[r][a] = 0.f;
      if (j < L) {
#pragma unroll
        for (int cc = 0; cc < C::KCH; ++cc) {
          const uint8_t* krow = Ks + cc * C::CHUNK + gt * 128;
#pragma unroll
          for (int seg = 0; seg < 8; ++seg) {
            const uint4 kv = *reinterpret_cast<const uint4*>(krow + ((seg ^ (gt & 7)) << 4));
            const float2 k01 = unpack2<BF16>(kv.x), k23 = unpack2<BF16>(kv.y);
            const float2 k45 = unpack2<BF16>(kv.z), k67 = unpack2<BF16>(kv.w);
            const float kf[8] = {k01.x, k01.y, k23.x, k23.y, k45.x, k45.y, k67.x, k67.y};
#pragma unroll
            for (int r = 0; r < NQ; ++r) {
              if (r < Nq) {
                const float4 qa = *reinterpret_cast<const float4*>(qs + r * D + cc * 64 + seg * 8);
                const float4 qb =
                    *reinterpret_cast<const float4*>(qs + r * D + cc * 64 + seg * 8 + 4);
                const float qf[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
                if constexpr (!PAIRED) {
#pragma unroll
                  for (int e = 0; e < 8; ++e)
                    acc[r][e % NACC] = fmaf(qf[e], kf[e], acc[r][e % NACC]);
                } else {
                  // two lanes per instruction (fma.rn.f32x2): element e still goes to
                  // partial sum e % NACC, so the sums are those of the scalar form
#pragma unroll
                  for (int e = 0; e < 8; e += 2) {
                    const int a = e % NACC;
                    const float2 t = f2_unpack(f2_fma(f2_pack(qf[e], qf[e + 1]),
                                                      f2_pack(kf[e], kf[e + 1]),
                                                      f2_pack(acc[r][a], acc[r][a + 1])));
                    acc[r][a] = t.x;
                    acc[r][a + 1] = t.y;
                  }
                }
              }
            }
          }
        }
      }
#pragma unroll
      for (int r = 0; r < NQ; ++r) {
        float a = 0.f;
#pragma unroll
        for (int v = 0; v < NACC; ++v) a += acc[r][v];
        const int pos = L - Nq + r;  // this query row's position in the sequence
        const bool ok =
            r < Nq && j < L && (wr < 0 || j <= pos + wr) && (wl < 0 || j >= pos - wl);
        x[r] = ok ? a * c : -INFINITY;
      }
    }
    // ---- tile maximum per row: warp shuffles, then the group's four warps in shared memory
#pragma unroll
    for (int r = 0; r < NQ; ++r) {
      if (r < Nq) {
        float mx = x[r];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) WMb[gw * NQ + r] = mx;
      }
    }
    named_barrier_sync(gbar, 128);
    // ---- p = 2^(x - m_new) for this thread's key; alpha rescales l and O
    float alpha[NQ];
#pragma unroll
    for (int r = 0; r < NQ; ++r) {
      alpha[r] = 1.f;
      if (r < Nq) {
        const float mt = fmaxf(fmaxf(WMb[r], WMb[NQ + r]), fmaxf(WMb[2 * NQ + r], WMb[3 * NQ + r]));
        const float m_new = fmaxf(m_run[r], mt);
        const float mu = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[r] = ex2_approx(m_run[r] - mu);  // 0 while the row had no key yet
        const float pr = ex2_approx(x[r] - mu);
        l_run[r] = l_run[r] * alpha[r] + pr;
        m_run[r] = m_new;
        Sb[r * BN + gt] = pr;
      }
    }
    named_barrier_sync(gbar, 128);

    // ---- O = alpha·O + P V (warp = 32 keys, lane = CPL columns); keys past L skipped
    mbar_wait(BAR(B_VFULL + s), ph, abort_flag, p.status);
#pragma unroll
    for (int r = 0; r < NQ; ++r) {
      if (r < Nq) {
        if constexpr (!PAIRED) {
#pragma unroll
          for (int e = 0; e < CPL; ++e) o[r][e] *= alpha[r];
        } else {
#pragma unroll
          for (int e = 0; e < CPL; e += 2) {
            const float2 t = f2_unpack(f2_mul(f2_pack(o[r][e], o[r][e + 1]),
                                              f2_pack(alpha[r], alpha[r])));
            o[r][e] = t.x;
            o[r][e + 1] = t.y;
          }
        }
      }
    }
    const uint8_t* vcol = Vs + vchunk * C::CHUNK + vbyte;
    const int jb = gw * 32;
    const int je = min(jb + 32, L - k0);
    auto pv_key = [&](int jj) {
      const uint8_t* vp = vcol + jj * 128 + ((vseg ^ (jj & 7)) << 4);
      float vf[CPL];
      if constexpr (CPL == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(vp);
        const float2 a = unpack2<BF16>(w.x), bb = unpack2<BF16>(w.y);
        vf[0] = a.x; vf[1] = a.y; vf[2] = bb.x; vf[3] = bb.y;
      } else {
        const float2 a = unpack2<BF16>(*reinterpret_cast<const uint32_t*>(vp));
        vf[0] = a.x; vf[1] = a.y;
      }
#pragma unroll
      for (int r = 0; r < NQ; ++r) {
        if (r < Nq) {
          const float pr = Sb[r * BN + jj];
          if constexpr (!PAIRED) {
#pragma unroll
            for (int e = 0; e < CPL; ++e) o[r][e] = fmaf(pr, vf[e], o[r][e]);
          } else {
#pragma unroll
            for (int e = 0; e < CPL; e += 2) {
              const float2 t = f2_unpack(f2_fma(f2_pack(pr, pr), f2_pack(vf[e], vf[e + 1]),
                                                f2_pack(o[r][e], o[r][e + 1])));
              o[r][e] = t.x;
              o[r][e + 1] = t.y;
            }
          }
        }
      }
    };
    if (je == jb + 32) {
#pragma unroll 8
      for (int jj = jb; jj < jb + 32; ++jj) pv_key(jj);
    } else {
      for (int jj = jb; jj < je; ++jj) pv_key(jj);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(BAR(B_EMPTY + s));
  }

  // ---- merge: groups' maxima, then the warps' partial O and the threads' partial l, each
  // weighted by 2^(m_group - M) (exactly 1 for a single group)
  named_barrier_sync(3, NCOMP);  // every tile consumed: the ring may be reused
  float* red = reinterpret_cast<float*>(sgen);  // [G][4][NQ][D] over the drained K/V ring
#pragma unroll
  for (int r = 0; r < NQ; ++r) {
    if (r < Nq) {
#pragma unroll
      for (int e = 0; e < CPL; ++e) red[((g * 4 + gw) * NQ + r) * D + col0 + e] = o[r][e];
      float l = l_run[r];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
      if (lane == 0) LW[gw * NQ + r] = l;
      if (gt == 0) MG[g * NQ + r] = m_run[r];
    }
  }
  named_barrier_sync(3, NCOMP);
  float* LWall = reinterpret_cast<float*>(sgen + C::OFF_L);
  for (int e = tid; e < Nq * D; e += NCOMP) {
    const int r = e / D, cc = e - r * D;
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < G; ++q) M = fmaxf(M, MG[q * NQ + r]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float sum = 0.f, l = 0.f;
#pragma unroll
    for (int q = 0; q < G; ++q) {
      const float wq = ex2_approx(MG[q * NQ + r] - Mu);  // 0 for a group that saw no key
      const float* rq = red + (q * 4 * NQ + r) * D + cc;
      sum += wq * ((rq[0] + rq[NQ * D]) + (rq[2 * NQ * D] + rq[3 * NQ * D]));
      const float* lq = LWall + q * 4 * NQ + r;
      l += wq * ((lq[0] + lq[NQ]) + (lq[2 * NQ] + lq[3 * NQ]));
    }
    const float val = l > 0.f ? sum / l : 0.f;
    if (p.splits == 1) {
      uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) + ((size_t)(b * Nq + r) * p.H + h) * D;
      orow[cc] = (uint16_t)(pack2<BF16>(val, 0.f) & 0xFFFFu);
      if (cc == 0)
        p.lse[((size_t)b * p.H + h) * Nq + r] =
            l > 0.f ? (M + lg2_approx(l)) * 0.69314718055994530942f : INFINITY;
    } else {
      const size_t row = ((size_t)(b * Nq + r) * p.H + h) * p.splits + split;
      p.o_part[row * D + cc] = val;
      if (cc == 0) p.lse_part[row] = l > 0.f ? M + lg2_approx(l) : -INFINITY;
    }
  }
}

// Merge of the splits' partial results, one warp per (sequence, query row, head).
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_decode_combine_kernel(const DecParams p) {
  constexpr int CPL = D / 32;
  const int gw = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= p.B * p.Nq * p.H) return;
  const int S = p.splits;
  const float* lp = p.lse_part + (size_t)gw * S;
  float M = -INFINITY;
  for (int s = lane; s < S; s += 32) M = fmaxf(M, lp[s]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const int h = gw % p.H, br = gw / p.H;
  const int r = br % p.Nq, b = br / p.Nq;
  uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) + (size_t)gw * D + lane * CPL;
  float* lse = p.lse + ((size_t)b * p.H + h) * p.Nq + r;
  if (M == -INFINITY) {  // no split saw a key: O = 0, LSE = +inf
#pragma unroll
    for (int e = 0; e < CPL; ++e) orow[e] = 0;
    if (lane == 0) *lse = INFINITY;
    return;
  }
  float W = 0.f;
  for (int s = lane; s < S; s += 32) W += ex2_approx(lp[s] - M);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) W += __shfl_xor_sync(0xffffffffu, W, off);
  float acc[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) acc[e] = 0.f;
  for (int s = 0; s < S; ++s) {
    const float w = ex2_approx(lp[s] - M);
    const float* op = p.o_part + ((size_t)gw * S + s) * D + lane * CPL;
    if constexpr (CPL == 4) {
      const float4 v = *reinterpret_cast<const float4*>(op);
      acc[0] = fmaf(w, v.x, acc[0]);
      acc[1] = fmaf(w, v.y, acc[1]);
      acc[2] = fmaf(w, v.z, acc[2]);
      acc[3] = fmaf(w, v.w, acc[3]);
    } else {
      const float2 v = *reinterpret_cast<const float2*>(op);
      acc[0] = fmaf(w, v.x, acc[0]);
      acc[1] = fmaf(w, v.y, acc[1]);
    }
  }
  const float inv = 1.f / W;
  if constexpr (CPL == 4) {
    *reinterpret_cast<uint2*>(orow) =
        make_uint2(pack2<BF16>(acc[0] * inv, acc[1] * inv), pack2<BF16>(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(orow) = pack2<BF16>(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0) *lse = (M + lg2_approx(W)) * 0.69314718055994530942f;
}

}  // namespace fattn
