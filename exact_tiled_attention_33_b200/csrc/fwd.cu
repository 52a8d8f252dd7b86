// Forward kernel instantiations and launchers.
#include <mutex>

#include "fwd_kernel.cuh"

namespace fattn {

int fwd_rows_per_cta(bool fp8) { return fp8 ? FwdCfg<128, true>::BM : FwdCfg<128>::BM; }

template <int D, bool BF16, bool FP8 = false, bool F32O = false, bool PACKED = false>
static LaunchResult launch_fwd_t(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                 const CUtensorMap& tmV, const CUtensorMap& tmO,
                                 const FwdParams& p, dim3 grid, cudaStream_t stream) {
  using C = FwdCfg<D, FP8>;
  auto kern = fa_fwd_kernel<D, BF16, FP8, F32O, PACKED>;
  static std::once_flag once[64];
  static cudaError_t set_err[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LaunchResult::kCudaError;
  if (dev < 0 || dev >= 64) return launch_status(cudaErrorInvalidDevice);
  std::call_once(once[dev], [&] {
    set_err[dev] =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  });
  if (set_err[dev] != cudaSuccess) return launch_status(set_err[dev]);
  kern<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tmQ, tmK, tmV, tmO, p);
  return launch_status(cudaGetLastError());
}

// the packed varlen grid takes its own kernel instance
template <int D, bool BF16, bool FP8 = false>
static LaunchResult launch_fwd_grid(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                    const CUtensorMap& tmV, const CUtensorMap& tmO,
                                    const FwdParams& p, dim3 grid, cudaStream_t stream) {
  return p.packed ? launch_fwd_t<D, BF16, FP8, false, true>(tmQ, tmK, tmV, tmO, p, grid, stream)
                  : launch_fwd_t<D, BF16, FP8, false, false>(tmQ, tmK, tmV, tmO, p, grid, stream);
}

LaunchResult launch_fwd(int d, bool bf16, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                        const CUtensorMap& tmV, const CUtensorMap& tmO, const FwdParams& p,
                        dim3 grid, cudaStream_t stream) {
  if (d == 128) {
    return bf16 ? launch_fwd_grid<128, true>(tmQ, tmK, tmV, tmO, p, grid, stream)
                : launch_fwd_grid<128, false>(tmQ, tmK, tmV, tmO, p, grid, stream);
  }
  if (d == 64) {
    return bf16 ? launch_fwd_grid<64, true>(tmQ, tmK, tmV, tmO, p, grid, stream)
                : launch_fwd_grid<64, false>(tmQ, tmK, tmV, tmO, p, grid, stream);
  }
  return LaunchResult::kUnsupported;
}

LaunchResult launch_fwd_fp8(int d, bool bf16, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                            const CUtensorMap& tmV, const CUtensorMap& tmO, const FwdParams& p,
                            dim3 grid, cudaStream_t stream) {
  if (d != 128) return LaunchResult::kUnsupported;
  return bf16 ? launch_fwd_grid<128, true, true>(tmQ, tmK, tmV, tmO, p, grid, stream)
              : launch_fwd_grid<128, false, true>(tmQ, tmK, tmV, tmO, p, grid, stream);
}

LaunchResult launch_fwd_f32out(int d, bool bf16, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                               const CUtensorMap& tmV, const CUtensorMap& tmO, const FwdParams& p,
                               dim3 grid, cudaStream_t stream) {
  if (d == 128)
    return bf16 ? launch_fwd_t<128, true, false, true>(tmQ, tmK, tmV, tmO, p, grid, stream)
                : launch_fwd_t<128, false, false, true>(tmQ, tmK, tmV, tmO, p, grid, stream);
  if (d == 64)
    return bf16 ? launch_fwd_t<64, true, false, true>(tmQ, tmK, tmV, tmO, p, grid, stream)
                : launch_fwd_t<64, false, false, true>(tmQ, tmK, tmV, tmO, p, grid, stream);
  return LaunchResult::kUnsupported;
}

}  // namespace fattn
