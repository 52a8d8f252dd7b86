// KV-cache decode kernel instantiations and launcher.
#include <mutex>

#include "decode_kernel.cuh"

namespace fattn {

template <int D, bool BF16, bool PAGED, int NQ>
static LaunchResult launch_decode_t(const CUtensorMap& tmK, const CUtensorMap& tmV,
                                    const DecParams& p, cudaStream_t stream) {
  using C = DecCfg<D, NQ>;
  auto kern = fa_decode_kernel<D, BF16, PAGED, NQ>;
  static std::once_flag once[64];
  static cudaError_t set_err[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LaunchResult::kCudaError;
  if (dev < 0 || dev >= 64) return launch_status(cudaErrorInvalidDevice);
  std::call_once(once[dev], [&] {
    set_err[dev] =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  });
  if (set_err[dev] != cudaSuccess) return launch_status(set_err[dev]);
  kern<<<dim3(p.splits, p.H, p.B), C::THREADS, C::SMEM_BYTES, stream>>>(tmK, tmV, p);
  if (p.splits > 1) {
    const long long warps = (long long)p.B * p.Nq * p.H;
    fa_decode_combine_kernel<D, BF16><<<(unsigned)((warps + 7) / 8), 256, 0, stream>>>(p);
  }
  return launch_status(cudaGetLastError());
}

template <int D, bool BF16, bool PAGED>
static LaunchResult launch_decode_nq(const CUtensorMap& tmK, const CUtensorMap& tmV,
                                     const DecParams& p, cudaStream_t stream) {
  if (p.Nq <= 1) return launch_decode_t<D, BF16, PAGED, 1>(tmK, tmV, p, stream);
  if (p.Nq <= 4) return launch_decode_t<D, BF16, PAGED, 4>(tmK, tmV, p, stream);
  if (p.Nq <= kDecodeMaxQueries)
    return launch_decode_t<D, BF16, PAGED, kDecodeMaxQueries>(tmK, tmV, p, stream);
  return LaunchResult::kUnsupported;
}

template <int D, bool BF16>
static LaunchResult launch_decode_paged(bool paged, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                        const DecParams& p, cudaStream_t stream) {
  return paged ? launch_decode_nq<D, BF16, true>(tmK, tmV, p, stream)
               : launch_decode_nq<D, BF16, false>(tmK, tmV, p, stream);
}

LaunchResult launch_decode(int d, bool bf16, bool paged, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const DecParams& p, cudaStream_t stream) {
  if (d == 128)
    return bf16 ? launch_decode_paged<128, true>(paged, tmK, tmV, p, stream)
                : launch_decode_paged<128, false>(paged, tmK, tmV, p, stream);
  if (d == 64)
    return bf16 ? launch_decode_paged<64, true>(paged, tmK, tmV, p, stream)
                : launch_decode_paged<64, false>(paged, tmK, tmV, p, stream);
  return LaunchResult::kUnsupported;
}

}  // namespace fattn
