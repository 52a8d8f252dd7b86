// Backward kernel instantiations and launcher: D preprocess, then the dK/dV pass and the
// dQ pass, all on the caller's stream.
#include <algorithm>
#include <mutex>

#include "bwd_fused_kernel.cuh"
#include "bwd_kernel.cuh"

namespace fattn {

template <int D, bool BF16>
static LaunchResult launch_bwd_t(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                 const CUtensorMap& tmV, const CUtensorMap& tmDO,
                                 const BwdParams& p, long long q_rows, int max_seqlen_q,
                                 int max_seqlen_k, int batches, cudaStream_t stream) {
  using C = BwdCfg<D>;
  static std::once_flag once[64];
  static cudaError_t set_err[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LaunchResult::kCudaError;
  if (dev < 0 || dev >= 64) return launch_status(cudaErrorInvalidDevice);
  std::call_once(once[dev], [&] {
    set_err[dev] = cudaFuncSetAttribute(fa_bwd_dkdv_kernel<D, BF16>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_A);
    if (set_err[dev] == cudaSuccess)
      set_err[dev] = cudaFuncSetAttribute(fa_bwd_dq_kernel<D, BF16>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_B);
  });
  if (set_err[dev] != cudaSuccess) return launch_status(set_err[dev]);
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // 1) D = rowsum(dO ∘ O)
  const long long warps = q_rows * p.H;
  const long long pre_blocks = std::min<long long>((warps + 7) / 8, (long long)sms * 16);
  fa_bwd_pre_kernel<D, BF16><<<(unsigned)pre_blocks, 256, 0, stream>>>(p, q_rows);
  // 2) dK, dV: one CTA per key tile
  dim3 grid_a((max_seqlen_k + C::BN - 1) / C::BN, p.H, batches);
  fa_bwd_dkdv_kernel<D, BF16><<<grid_a, C::THREADS, C::SMEM_A, stream>>>(tmQ, tmK, tmV, tmDO, p);
  // 3) dQ: one CTA per query tile
  dim3 grid_b((max_seqlen_q + C::BM - 1) / C::BM, p.H, batches);
  fa_bwd_dq_kernel<D, BF16><<<grid_b, C::THREADS, C::SMEM_B, stream>>>(tmQ, tmK, tmV, tmDO, p);
  return launch_status(cudaGetLastError());
}

template <int D, bool BF16, bool PACKED>
static LaunchResult launch_bwd_fused_t(const BwdFusedMaps& m, const BwdParams& p,
                                       long long q_rows, int max_seqlen_k, int batches,
                                       cudaStream_t stream) {
  using C = BwdFusedCfg<D>;
  static std::once_flag once[64];
  static cudaError_t set_err[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LaunchResult::kCudaError;
  if (dev < 0 || dev >= 64) return launch_status(cudaErrorInvalidDevice);
  std::call_once(once[dev], [&] {
    set_err[dev] = cudaFuncSetAttribute(fa_bwd_fused_kernel<D, BF16, PACKED>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  });
  if (set_err[dev] != cudaSuccess) return launch_status(set_err[dev]);
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // 1) D = rowsum(dO ∘ O) and zeroed dQ sums
  const long long warps = q_rows * p.H;
  const long long pre_blocks = std::min<long long>((warps + 7) / 8, (long long)sms * 16);
  fa_bwd_pre_acc_kernel<D, BF16><<<(unsigned)pre_blocks, 256, 0, stream>>>(p, q_rows);
  // 2) dK, dV and the dQ partial sums: one CTA per key tile
  //    (a packed varlen grid numbers the key tiles of all sequences: see packed_tile_lookup)
  static_assert(C::BN == 128, "the packed grid's tiles are 128 keys");
  const dim3 grid =
      PACKED ? dim3((unsigned)packed_grid_tiles(p.total_k, batches, max_seqlen_k), p.H, 1)
             : dim3((max_seqlen_k + C::BN - 1) / C::BN, p.H, batches);
  //    (a programmatic dependent of the preprocess: see grid_dependency_wait in the kernel)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, fa_bwd_fused_kernel<D, BF16, PACKED>, m.q, m.k, m.v,
                                     m.dout, m.dq, m.dk, m.dv, p);
  if (e != cudaSuccess) return launch_status(e);
  // 3) dQ = scale * sums, rounded to 16 bits
  const long long elems = q_rows * p.H * D;
  const long long cv_blocks = std::min<long long>((elems / 8 + 255) / 256, (long long)sms * 16);
  //    (a programmatic dependent of the fused pass)
  cfg.gridDim = dim3((unsigned)cv_blocks);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&cfg, fa_bwd_dq_convert_kernel<BF16>, p, elems);
  if (e != cudaSuccess) return launch_status(e);
  return launch_status(cudaGetLastError());
}

// the packed varlen grid takes its own kernel instance
template <int D, bool BF16>
static LaunchResult launch_bwd_fused_grid(const BwdFusedMaps& m, const BwdParams& p,
                                          long long q_rows, int max_seqlen_k, int batches,
                                          cudaStream_t stream) {
  return p.packed
             ? launch_bwd_fused_t<D, BF16, true>(m, p, q_rows, max_seqlen_k, batches, stream)
             : launch_bwd_fused_t<D, BF16, false>(m, p, q_rows, max_seqlen_k, batches, stream);
}

LaunchResult launch_bwd_fused(int d, bool bf16, const BwdFusedMaps& m, const BwdParams& p,
                              long long q_rows, int max_seqlen_k, int batches,
                              cudaStream_t stream) {
  if (d == 128)
    return bf16 ? launch_bwd_fused_grid<128, true>(m, p, q_rows, max_seqlen_k, batches, stream)
                : launch_bwd_fused_grid<128, false>(m, p, q_rows, max_seqlen_k, batches, stream);
  if (d == 64)
    return bf16 ? launch_bwd_fused_grid<64, true>(m, p, q_rows, max_seqlen_k, batches, stream)
                : launch_bwd_fused_grid<64, false>(m, p, q_rows, max_seqlen_k, batches, stream);
  return LaunchResult::kUnsupported;
}

LaunchResult launch_bwd(int d, bool bf16, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                        const CUtensorMap& tmV, const CUtensorMap& tmDO, const BwdParams& p,
                        long long q_rows, int max_seqlen_q, int max_seqlen_k, int batches,
                        cudaStream_t stream) {
  if (d == 128)
    return bf16 ? launch_bwd_t<128, true>(tmQ, tmK, tmV, tmDO, p, q_rows, max_seqlen_q, max_seqlen_k, batches, stream)
                : launch_bwd_t<128, false>(tmQ, tmK, tmV, tmDO, p, q_rows, max_seqlen_q, max_seqlen_k, batches, stream);
  if (d == 64)
    return bf16 ? launch_bwd_t<64, true>(tmQ, tmK, tmV, tmDO, p, q_rows, max_seqlen_q, max_seqlen_k, batches, stream)
                : launch_bwd_t<64, false>(tmQ, tmK, tmV, tmDO, p, q_rows, max_seqlen_q, max_seqlen_k, batches, stream);
  return LaunchResult::kUnsupported;
}

}  // namespace fattn
