// C ABI of libfattn: argument validation, TMA tensor-map encoding, launches, status.
// The operations are documented in include/fattn.h.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "fattn.h"
#include "fattn_internal.h"
#include "sm100.cuh"

namespace fattn {

// One status word per device (each device that loads the module gets its own copy).
__device__ uint32_t g_status_word;

cudaError_t& launch_error() {
  static thread_local cudaError_t e = cudaSuccess;
  return e;
}

namespace {

thread_local std::string g_last_error;

int fail(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(FA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor-map encoding is a driver call and needs a current context on the calling
// thread.  A host thread that has made no CUDA runtime call yet (an autograd worker
// thread, for instance) has none; make the runtime's primary context current then.
int ensure_context() {
  using CtxGetCurrentFn = CUresult (*)(CUcontext*);
  static CtxGetCurrentFn get_current = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext ctx = nullptr;
  if (get_current != nullptr && get_current(&ctx) == CUDA_SUCCESS && ctx != nullptr) return FA_OK;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaSetDevice(dev);  // initialises and binds the primary context
  return e == cudaSuccess ? FA_OK : cuda_fail(e, "making the device context current");
}

// Tensor map over a [batches, rows, H, d] tensor of 16-bit (elem_bytes 2) or 8-bit
// (elem_bytes 1) elements, dims listed innermost first (d, H, rows, batches); box = one
// 128-byte swizzle row of d (64 or 128 elements) x 1 head x box_rows rows.  Out-of-range
// rows read as zero.
int make_map(CUtensorMap* map, const void* base, int d, int H, long long rows, long long batches,
             int box_rows, int elem_bytes = 2) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  if (int e = ensure_context()) return e;
  const cuuint64_t eb = (cuuint64_t)elem_bytes;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)batches};
  cuuint64_t strides[3] = {(cuuint64_t)d * eb, (cuuint64_t)H * d * eb,
                           (cuuint64_t)rows * H * d * eb};
  cuuint32_t box[4] = {(cuuint32_t)(128 / elem_bytes), 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt =
      elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
  CUresult r = enc(map, dt, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")");
  return FA_OK;
}

// Device address of a module variable on the current device, looked up once per device
// (std::call_once, so concurrent first calls from several host threads are safe).  The
// host-side symbol is only a stand-in and must never be handed to a kernel.
template <typename T>
struct PerDeviceSymbol {
  static constexpr int kMaxDevices = 64;
  std::once_flag once[kMaxDevices];
  T* ptr[kMaxDevices] = {};
  cudaError_t err[kMaxDevices] = {};
  // Returns the address (nullptr on failure, with the lookup's error in *e).
  template <typename Sym>
  T* get(const Sym& sym, int dev, cudaError_t* e) {
    if (dev < 0 || dev >= kMaxDevices) {
      *e = cudaErrorInvalidDevice;
      return nullptr;
    }
    std::call_once(once[dev], [&] {
      void* p = nullptr;
      err[dev] = cudaGetSymbolAddress(&p, sym);
      if (err[dev] == cudaSuccess) ptr[dev] = static_cast<T*>(p);
    });
    *e = err[dev];
    return ptr[dev];
  }
};

// Tensor map over fp32 [rows, H, d] sums for TMA reduce-adds: box 32 columns (128 bytes,
// one swizzle row) x 1 head x 128 rows, 128-byte swizzle; rows past the end are skipped.
int make_map_f32_reduce(CUtensorMap* map, float* base, int d, int H, long long rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  if (int e = ensure_context()) return e;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)rows, 1};
  cuuint64_t strides[3] = {(cuuint64_t)d * 4, (cuuint64_t)H * d * 4, (cuuint64_t)rows * H * d * 4};
  cuuint32_t box[4] = {32, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled (dQ sums) failed (code " + std::to_string((int)r) + ")");
  return FA_OK;
}

uint32_t* status_ptr() {
  static PerDeviceSymbol<uint32_t> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  cudaError_t e = cudaSuccess;
  return cache.get(g_status_word, dev, &e);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int H, int d, int dtype, float scale) {
  if (H < 0 || H > 65535) return fail(FA_ERR_UNSUPPORTED, "H must be in [0, 65535]");
  if (d != 64 && d != 128) return fail(FA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (dtype != FA_BF16 && dtype != FA_FP16) return fail(FA_ERR_UNSUPPORTED, "unknown dtype");
  if (!std::isfinite(scale)) return fail(FA_ERR_INVALID_ARG, "scale must be finite");
  return FA_OK;
}

int check_ptrs(std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs) {
    if (p == nullptr) return fail(FA_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(p)) return fail(FA_ERR_INVALID_ARG, "pointer not 16-byte aligned");
  }
  return FA_OK;
}

// Grids are x = 128-row tiles of the sequence, y = heads, z = batches or sequences.
int check_grid(long long batches, long long H, long long max_len) {
  if (batches > 65535) return fail(FA_ERR_UNSUPPORTED, "batch / number of sequences must be <= 65535");
  if (H > 65535) return fail(FA_ERR_UNSUPPORTED, "H must be <= 65535");
  (void)max_len;  // B*N < 2^31 bounds the tile count far below the x-dimension limit
  return FA_OK;
}

int launch_result(LaunchResult r) {
  if (r == LaunchResult::kOk) return FA_OK;
  if (r == LaunchResult::kUnsupported) return fail(FA_ERR_UNSUPPORTED, "unsupported configuration");
  const cudaError_t e = launch_error() != cudaSuccess ? launch_error() : cudaGetLastError();
  launch_error() = cudaSuccess;
  return cuda_fail(e, "kernel launch");
}

constexpr float kLog2e = 1.4426950408889634f;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// The forward kernel works with a positive log2-domain factor c: a negative scale is
// applied by negating Q in the S product, and scale == 0 uses a factor so small that
// every finite score maps to x = 0 exactly in fp32 (uniform weights) while masked
// scores (-inf) stay -inf.
void set_fwd_scale(FwdParams& p, float scale) {
  p.v_descale = 1.f;
  p.negate_scores = scale < 0.f ? 1 : 0;
  const float c = std::fabs(scale) * kLog2e;
  p.scale_log2 = c > 1e-30f ? c : 1e-30f;
}

// Attention window arguments: any negative bound means "no bound" (-1); a bound that
// already admits every key of every sequence (right >= max_seqlen_q - 1, left >=
// max_seqlen_k - 1) becomes -1 too, so the kernels only see bounds below the sequence
// lengths.  Index sums stay in int32 when max_seqlen_q + max_seqlen_k < 2^31.
int normalize_window(int* wl, int* wr, long long max_q, long long max_k) {
  if (*wl < 0) *wl = -1;
  if (*wr < 0) *wr = -1;
  if (*wr >= 0 && (long long)*wr >= max_q - 1) *wr = -1;
  if (*wl >= 0 && (long long)*wl >= max_k - 1) *wl = -1;
  if ((*wl >= 0 || *wr > 0) && max_q + max_k >= (1LL << 31))
    return fail(FA_ERR_UNSUPPORTED, "windowed attention needs max_seqlen_q + max_seqlen_k < 2^31");
  return FA_OK;
}

// Causal-style windows (no left bound) give the last query tiles the most key tiles;
// those are launched first.
int reverse_tiles(int wl, int wr) { return (wl < 0 && wr >= 0) ? 1 : 0; }

// Grid of a varlen forward: per sequence (x = query tiles of the longest sequence, z =
// sequences), or packed (x = the query tiles of all sequences) when that launches far fewer
// CTAs (use_packed_grid; its tiles are 128 rows, as are the forward's).
dim3 varlen_fwd_grid(FwdParams& p, int rows, int total_q, int num_seqs, int max_seqlen_q,
                     int H) {
  p.num_seqs = num_seqs;
  p.packed = (rows == 128 && use_packed_grid(total_q, num_seqs, max_seqlen_q)) ? 1 : 0;
  if (p.packed) return dim3((unsigned)packed_grid_tiles(total_q, num_seqs, max_seqlen_q), H, 1);
  return dim3((max_seqlen_q + rows - 1) / rows, H, num_seqs);
}

int fwd_dense(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N,
              int H, int d, float scale, int wl, int wr, int dtype, void* stream) {
  if (int e = check_common(H, d, dtype, scale)) return e;
  if (B < 0 || N < 0) return fail(FA_ERR_INVALID_ARG, "B and N must be >= 0");
  if ((long long)B * N >= (1LL << 31)) return fail(FA_ERR_UNSUPPORTED, "B*N must be < 2^31");
  if (B == 0 || N == 0 || H == 0) return FA_OK;
  if (int e = check_grid(B, H, N)) return e;
  if (int e = normalize_window(&wl, &wr, N, N)) return e;
  if (int e = check_ptrs({q, k, v, o, lse})) return e;
  CUtensorMap mq, mk, mv;
  if (int e = make_map(&mq, q, d, H, N, B, 128)) return e;
  if (int e = make_map(&mk, k, d, H, N, B, 128)) return e;
  if (int e = make_map(&mv, v, d, H, N, B, 128)) return e;
  CUtensorMap mo;  // O leaves through TMA stores
  if (int e = make_map(&mo, o, d, H, N, B, 128)) return e;
  FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.cu_q = p.cu_k = nullptr;
  p.N = N;
  p.H = H;
  p.total_q = B * N;
  p.scale = scale;
  set_fwd_scale(p, scale);
  p.win_left = wl;
  p.win_right = wr;
  p.reverse_tiles = reverse_tiles(wl, wr);
  p.max_seqlen_q = N;
  p.status = status_ptr();
  if (p.status == nullptr) return cuda_fail(cudaGetLastError(), "status word");
  const int rows = fwd_rows_per_cta(false);
  dim3 grid((N + rows - 1) / rows, H, B);
  return launch_result(
      launch_fwd(d, dtype == FA_BF16, mq, mk, mv, mo, p, grid, (cudaStream_t)stream));
}

int fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
               const int* cu_seqlens_q, const int* cu_seqlens_k, int max_seqlen_q,
               int max_seqlen_k, int H, int d, float scale, int wl, int wr, int num_seqs,
               int total_q, int total_k, int dtype, void* stream) {
  if (int e = check_common(H, d, dtype, scale)) return e;
  if (num_seqs < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0)
    return fail(FA_ERR_INVALID_ARG, "sizes must be >= 0");
  if (num_seqs > 65535) return fail(FA_ERR_UNSUPPORTED, "num_seqs must be <= 65535");
  if (max_seqlen_q > total_q || max_seqlen_k > total_k)
    return fail(FA_ERR_INVALID_ARG, "max_seqlen exceeds the total token count");
  if (num_seqs == 0 || total_q == 0 || H == 0 || max_seqlen_q == 0) return FA_OK;
  if (int e = check_grid(num_seqs, H, std::max(max_seqlen_q, max_seqlen_k))) return e;
  if (int e = normalize_window(&wl, &wr, max_seqlen_q, max_seqlen_k)) return e;
  if (int e = check_ptrs({q, o, lse, cu_seqlens_q, cu_seqlens_k})) return e;
  if (total_k > 0)
    if (int e = check_ptrs({k, v})) return e;
  CUtensorMap mq, mk, mv;
  if (int e = make_map(&mq, q, d, H, total_q, 1, 128)) return e;
  // With no keys at all every row is fully masked and K/V are never read.
  const void* kb = total_k > 0 ? k : q;
  const void* vb = total_k > 0 ? v : q;
  const long long kr = total_k > 0 ? total_k : total_q;
  if (int e = make_map(&mk, kb, d, H, kr, 1, 128)) return e;
  if (int e = make_map(&mv, vb, d, H, kr, 1, 128)) return e;
  CUtensorMap mo;
  if (int e = make_map(&mo, o, d, H, total_q, 1, 128)) return e;
  FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.N = 0;
  p.H = H;
  p.total_q = total_q;
  p.total_k = total_k;
  p.scale = scale;
  set_fwd_scale(p, scale);
  p.win_left = wl;
  p.win_right = wr;
  p.reverse_tiles = reverse_tiles(wl, wr);
  p.max_seqlen_q = max_seqlen_q;
  p.status = status_ptr();
  if (p.status == nullptr) return cuda_fail(cudaGetLastError(), "status word");
  const dim3 grid =
      varlen_fwd_grid(p, fwd_rows_per_cta(false), total_q, num_seqs, max_seqlen_q, H);
  return launch_result(
      launch_fwd(d, dtype == FA_BF16, mq, mk, mv, mo, p, grid, (cudaStream_t)stream));
}

}  // namespace

// Bounded-wait self test: waits on a barrier that nothing arrives at.
__global__ void selftest_wait_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  mbar_wait_limit(smem_u32(&bar), 0, &abort_flag, status, limit_ns);
}

// Evaluates the FMA-pipe exponential used by the forward softmax, for testing it against
// the hardware ex2 and against exact values.
__global__ void selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_poly2(x[i], x[i + 1]);
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly2(x[i], 0.f).x;
  }
}

}  // namespace fattn

using namespace fattn;

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N, int H,
           int d, float scale, int causal, int dtype, void* stream) {
  g_last_error.clear();
  return fwd_dense(q, k, v, o, lse, B, N, H, d, scale, -1, causal ? 0 : -1, dtype, stream);
}

int fa_fwd_local(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N,
                 int H, int d, float scale, int window_left, int window_right, int dtype,
                 void* stream) {
  g_last_error.clear();
  return fwd_dense(q, k, v, o, lse, B, N, H, d, scale, window_left, window_right, dtype, stream);
}

int fa_varlen_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int max_seqlen_q,
                  int max_seqlen_k, int H, int d, float scale, int causal, int num_seqs,
                  int total_q, int total_k, int dtype, void* stream) {
  g_last_error.clear();
  return fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, H,
                    d, scale, -1, causal ? 0 : -1, num_seqs, total_q, total_k, dtype, stream);
}

int fa_varlen_fwd_local(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int max_seqlen_q,
                        int max_seqlen_k, int H, int d, float scale, int window_left,
                        int window_right, int num_seqs, int total_q, int total_k, int dtype,
                        void* stream) {
  g_last_error.clear();
  return fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, H,
                    d, scale, window_left, window_right, num_seqs, total_q, total_k, dtype,
                    stream);
}

// ------------------------------------------------------------------ FP8 forward
namespace {

int fp8_check(int d, float scale, float q_descale, float k_descale, float v_descale,
              int out_dtype) {
  if (d != 128) return fail(FA_ERR_UNSUPPORTED, "FP8 forward takes head_dim 128");
  if (out_dtype != FA_BF16 && out_dtype != FA_FP16) return fail(FA_ERR_UNSUPPORTED, "unknown dtype");
  if (!std::isfinite(scale) || scale < 0.f)
    return fail(FA_ERR_UNSUPPORTED, "FP8 forward takes a finite scale >= 0");
  for (float s : {q_descale, k_descale, v_descale})
    if (!std::isfinite(s) || s <= 0.f)
      return fail(FA_ERR_INVALID_ARG, "descale factors must be finite and > 0");
  return FA_OK;
}

void set_fp8_scale(FwdParams& p, float scale, float q_descale, float k_descale,
                   float v_descale) {
  set_fwd_scale(p, scale * q_descale * k_descale);
  p.v_descale = v_descale;
}

}  // namespace

int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N,
               int H, int d, float scale, float q_descale, float k_descale, float v_descale,
               int causal, int out_dtype, void* stream) {
  g_last_error.clear();
  if (int e = fp8_check(d, scale, q_descale, k_descale, v_descale, out_dtype)) return e;
  if (H < 0 || H > 65535) return fail(FA_ERR_UNSUPPORTED, "H must be in [0, 65535]");
  if (B < 0 || N < 0) return fail(FA_ERR_INVALID_ARG, "B and N must be >= 0");
  if ((long long)B * N >= (1LL << 31)) return fail(FA_ERR_UNSUPPORTED, "B*N must be < 2^31");
  if (B == 0 || N == 0 || H == 0) return FA_OK;
  if (int e = check_grid(B, H, N)) return e;
  if (int e = check_ptrs({q, k, v, o, lse})) return e;
  CUtensorMap mq, mk, mv;
  if (int e = make_map(&mq, q, d, H, N, B, 128, 1)) return e;
  if (int e = make_map(&mk, k, d, H, N, B, 128, 1)) return e;
  if (int e = make_map(&mv, v, d, H, N, B, 128, 1)) return e;
  CUtensorMap mo;  // 16-bit O
  if (int e = make_map(&mo, o, d, H, N, B, 128)) return e;
  FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.N = N;
  p.H = H;
  p.total_q = B * N;
  p.scale = scale;
  set_fp8_scale(p, scale, q_descale, k_descale, v_descale);
  p.win_left = -1;
  p.win_right = causal ? 0 : -1;
  p.reverse_tiles = reverse_tiles(p.win_left, p.win_right);
  p.max_seqlen_q = N;
  p.status = status_ptr();
  if (p.status == nullptr) return cuda_fail(cudaGetLastError(), "status word");
  const int rows = fwd_rows_per_cta(true);
  dim3 grid((N + rows - 1) / rows, H, B);
  return launch_result(
      launch_fwd_fp8(d, out_dtype == FA_BF16, mq, mk, mv, mo, p, grid, (cudaStream_t)stream));
}

int fa_varlen_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                      const int* cu_seqlens_q, const int* cu_seqlens_k, int max_seqlen_q,
                      int max_seqlen_k, int H, int d, float scale, float q_descale,
                      float k_descale, float v_descale, int causal, int num_seqs, int total_q,
                      int total_k, int out_dtype, void* stream) {
  g_last_error.clear();
  if (int e = fp8_check(d, scale, q_descale, k_descale, v_descale, out_dtype)) return e;
  if (H < 0 || H > 65535) return fail(FA_ERR_UNSUPPORTED, "H must be in [0, 65535]");
  if (num_seqs < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0)
    return fail(FA_ERR_INVALID_ARG, "sizes must be >= 0");
  if (num_seqs > 65535) return fail(FA_ERR_UNSUPPORTED, "num_seqs must be <= 65535");
  if (max_seqlen_q > total_q || max_seqlen_k > total_k)
    return fail(FA_ERR_INVALID_ARG, "max_seqlen exceeds the total token count");
  if (num_seqs == 0 || total_q == 0 || H == 0 || max_seqlen_q == 0) return FA_OK;
  if (int e = check_grid(num_seqs, H, std::max(max_seqlen_q, max_seqlen_k))) return e;
  if (int e = check_ptrs({q, o, lse, cu_seqlens_q, cu_seqlens_k})) return e;
  if (total_k > 0)
    if (int e = check_ptrs({k, v})) return e;
  CUtensorMap mq, mk, mv;
  if (int e = make_map(&mq, q, d, H, total_q, 1, 128, 1)) return e;
  const void* kb = total_k > 0 ? k : q;
  const void* vb = total_k > 0 ? v : q;
  const long long kr = total_k > 0 ? total_k : total_q;
  if (int e = make_map(&mk, kb, d, H, kr, 1, 128, 1)) return e;
  if (int e = make_map(&mv, vb, d, H, kr, 1, 128, 1)) return e;
  CUtensorMap mo;  // 16-bit O
  if (int e = make_map(&mo, o, d, H, total_q, 1, 128)) return e;
  FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.H = H;
  p.total_q = total_q;
  p.total_k = total_k;
  p.scale = scale;
  set_fp8_scale(p, scale, q_descale, k_descale, v_descale);
  p.win_left = -1;
  p.win_right = causal ? 0 : -1;
  p.reverse_tiles = reverse_tiles(p.win_left, p.win_right);
  p.max_seqlen_q = max_seqlen_q;
  p.status = status_ptr();
  if (p.status == nullptr) return cuda_fail(cudaGetLastError(), "status word");
  const dim3 grid =
      varlen_fwd_grid(p, fwd_rows_per_cta(true), total_q, num_seqs, max_seqlen_q, H);
  return launch_result(
      launch_fwd_fp8(d, out_dtype == FA_BF16, mq, mk, mv, mo, p, grid, (cudaStream_t)stream));
}

namespace {

// Backward workspace: D = rowsum(dO ∘ O) (fp32, one per token row and head), then, for the
// single-pass backward, the fp32 dQ sums (H x rows rounded up to 32 x d).
size_t d_vector_bytes(long long rows, long long H) { return align256((size_t)rows * H * 4); }
size_t dq_sum_bytes(long long rows, long long H, long long d) {
  return align256((size_t)rows * H * d * 4);
}

}  // namespace

size_t fa_bwd_workspace_size(int B, int N, int H, int d) {
  if (B <= 0 || N <= 0 || H <= 0 || d <= 0) return 0;
  const long long rows = (long long)B * N;
  return d_vector_bytes(rows, H) + dq_sum_bytes(rows, H, d);
}

size_t fa_varlen_bwd_workspace_size(int total_q, int H, int d) {
  if (total_q <= 0 || H <= 0 || d <= 0) return 0;
  return d_vector_bytes(total_q, H) + dq_sum_bytes(total_q, H, d);
}

namespace {

// Shared validation and launch for both backward entry points.
int bwd_common(const void* q, const void* k, const void* v, const void* o, const void* dout,
               const float* lse, void* dq, void* dk, void* dv, const int* cu_q, const int* cu_k,
               int H, int d, float scale, int wl, int wr, long long q_rows, long long k_rows,
               int N, int batches, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
               void* workspace, size_t workspace_bytes, bool single_pass, int dtype,
               cudaStream_t stream) {
  const size_t need = d_vector_bytes(q_rows, H) + (single_pass ? dq_sum_bytes(q_rows, H, d) : 0);
  if (int e = normalize_window(&wl, &wr, max_seqlen_q, max_seqlen_k)) return e;
  if (int e = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv, workspace})) return e;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(FA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (workspace_bytes < need)
    return fail(FA_ERR_INVALID_ARG, "workspace too small (need " + std::to_string(need) + " bytes)");
  CUtensorMap mq, mk, mv, mdo;
  const long long qb = cu_q ? 1 : batches, kb = cu_q ? 1 : batches;
  const long long qr = cu_q ? q_rows : N, kr = cu_q ? k_rows : N;
  if (int e = make_map(&mq, q, d, H, qr, qb, 128)) return e;
  if (int e = make_map(&mdo, dout, d, H, qr, qb, 128)) return e;
  if (int e = make_map(&mk, k, d, H, kr, kb, 128)) return e;
  if (int e = make_map(&mv, v, d, H, kr, kb, 128)) return e;
  BwdParams p{};
  p.q = q; p.k = k; p.v = v; p.o = o; p.dout = dout; p.lse = lse;
  p.dq = dq; p.dk = dk; p.dv = dv;
  p.dvec = static_cast<float*>(workspace);
  p.dq_acc = single_pass ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                                    d_vector_bytes(q_rows, H))
                         : nullptr;
  p.cu_q = cu_q; p.cu_k = cu_k;
  p.B = cu_q ? 1 : batches; p.N = N; p.H = H;
  p.total_q = total_q; p.total_k = total_k;
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.win_left = wl;
  p.win_right = wr;
  p.reverse_tiles = reverse_tiles(wl, wr);
  p.max_seqlen_q = max_seqlen_q;
  p.max_seqlen_k = max_seqlen_k;
  p.num_seqs = cu_q ? batches : 0;
  // the single-pass kernel may take the packed grid over key tiles (use_packed_grid)
  p.packed = (cu_q && single_pass && use_packed_grid(total_k, batches, max_seqlen_k)) ? 1 : 0;
  p.status = status_ptr();
  if (p.status == nullptr) return cuda_fail(cudaGetLastError(), "status word");
  if (single_pass) {
    BwdFusedMaps m;
    m.q = mq; m.k = mk; m.v = mv; m.dout = mdo;
    // the fp32 dQ sums, [q_rows, H, d], reduce-added by the TMA unit 32 columns x 128 rows
    // at a time
    if (int e = make_map_f32_reduce(&m.dq, p.dq_acc, d, H, q_rows)) return e;
    if (int e = make_map(&m.dk, dk, d, H, kr, kb, 128)) return e;
    if (int e = make_map(&m.dv, dv, d, H, kr, kb, 128)) return e;
    return launch_result(
        launch_bwd_fused(d, dtype == FA_BF16, m, p, q_rows, max_seqlen_k, batches, stream));
  }
  return launch_result(launch_bwd(d, dtype == FA_BF16, mq, mk, mv, mdo, p, q_rows, max_seqlen_q,
                                  max_seqlen_k, batches, stream));
}

}  // namespace

namespace {

int bwd_dense(const void* q, const void* k, const void* v, const void* o, const void* dout,
              const float* lse, void* dq, void* dk, void* dv, int B, int N, int H, int d,
              float scale, int wl, int wr, void* workspace, size_t workspace_bytes,
              bool single_pass, int dtype, void* stream) {
  if (int e = check_common(H, d, dtype, scale)) return e;
  if (B < 0 || N < 0) return fail(FA_ERR_INVALID_ARG, "B and N must be >= 0");
  if ((long long)B * N >= (1LL << 31)) return fail(FA_ERR_UNSUPPORTED, "B*N must be < 2^31");
  if (B == 0 || N == 0 || H == 0) return FA_OK;
  if (int e = check_grid(B, H, N)) return e;
  return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, nullptr, nullptr, H, d, scale, wl, wr,
                    (long long)B * N, (long long)B * N, N, B, N, N, B * N, B * N, workspace,
                    workspace_bytes, single_pass, dtype, (cudaStream_t)stream);
}

int bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout,
               const float* lse, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
               const int* cu_seqlens_k, int max_seqlen_q, int max_seqlen_k, int H, int d,
               float scale, int wl, int wr, int num_seqs, int total_q, int total_k,
               void* workspace, size_t workspace_bytes, bool single_pass, int dtype,
               void* stream) {
  if (int e = check_common(H, d, dtype, scale)) return e;
  if (num_seqs < 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0)
    return fail(FA_ERR_INVALID_ARG, "sizes must be >= 0");
  if (num_seqs > 65535) return fail(FA_ERR_UNSUPPORTED, "num_seqs must be <= 65535");
  if (max_seqlen_q > total_q || max_seqlen_k > total_k)
    return fail(FA_ERR_INVALID_ARG, "max_seqlen exceeds the total token count");
  if (num_seqs == 0 || H == 0 || (total_q == 0 && total_k == 0)) return FA_OK;
  if (total_q == 0 || total_k == 0) {
    // One side empty: every gradient that exists is zero.
    if (int e = check_ptrs({total_q ? dq : dk})) return e;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t err = cudaSuccess;
    if (total_q) err = cudaMemsetAsync(dq, 0, (size_t)total_q * H * d * 2, st);
    if (total_k && err == cudaSuccess) err = cudaMemsetAsync(dk, 0, (size_t)total_k * H * d * 2, st);
    if (total_k && err == cudaSuccess) err = cudaMemsetAsync(dv, 0, (size_t)total_k * H * d * 2, st);
    return err == cudaSuccess ? FA_OK : cuda_fail(err, "cudaMemsetAsync");
  }
  if (int e = check_grid(num_seqs, H, std::max(max_seqlen_q, max_seqlen_k))) return e;
  return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, H, d, scale,
                    wl, wr, total_q, total_k, 0, num_seqs, max_seqlen_q, max_seqlen_k, total_q,
                    total_k, workspace, workspace_bytes, single_pass, dtype,
                    (cudaStream_t)stream);
}

}  // namespace

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
           const float* lse, void* dq, void* dk, void* dv, int B, int N, int H, int d, float scale,
           int causal, void* workspace, size_t workspace_bytes, int dtype, void* stream) {
  g_last_error.clear();
  return bwd_dense(q, k, v, o, dout, lse, dq, dk, dv, B, N, H, d, scale, -1, causal ? 0 : -1,
                   workspace, workspace_bytes, true, dtype, stream);
}

int fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                         int N, int H, int d, float scale, int window_left, int window_right,
                         void* workspace, size_t workspace_bytes, int dtype, void* stream) {
  g_last_error.clear();
  return bwd_dense(q, k, v, o, dout, lse, dq, dk, dv, B, N, H, d, scale, window_left,
                   window_right, workspace, workspace_bytes, false, dtype, stream);
}

int fa_bwd_local(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, int B, int N, int H, int d,
                 float scale, int window_left, int window_right, void* workspace,
                 size_t workspace_bytes, int dtype, void* stream) {
  g_last_error.clear();
  return bwd_dense(q, k, v, o, dout, lse, dq, dk, dv, B, N, H, d, scale, window_left,
                   window_right, workspace, workspace_bytes, true, dtype, stream);
}

int fa_varlen_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                  const int* cu_seqlens_k, int max_seqlen_q, int max_seqlen_k, int H, int d,
                  float scale, int causal, int num_seqs, int total_q, int total_k,
                  void* workspace, size_t workspace_bytes, int dtype, void* stream) {
  g_last_error.clear();
  return bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                    max_seqlen_k, H, d, scale, -1, causal ? 0 : -1, num_seqs, total_q, total_k,
                    workspace, workspace_bytes, true, dtype, stream);
}

int fa_varlen_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                                const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                const int* cu_seqlens_q, const int* cu_seqlens_k,
                                int max_seqlen_q, int max_seqlen_k, int H, int d, float scale,
                                int window_left, int window_right, int num_seqs, int total_q,
                                int total_k, void* workspace, size_t workspace_bytes, int dtype,
                                void* stream) {
  g_last_error.clear();
  return bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                    max_seqlen_k, H, d, scale, window_left, window_right, num_seqs, total_q,
                    total_k, workspace, workspace_bytes, false, dtype, stream);
}

int fa_varlen_bwd_local(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int max_seqlen_q,
                        int max_seqlen_k, int H, int d, float scale, int window_left,
                        int window_right, int num_seqs, int total_q, int total_k,
                        void* workspace, size_t workspace_bytes, int dtype, void* stream) {
  g_last_error.clear();
  return bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                    max_seqlen_k, H, d, scale, window_left, window_right, num_seqs, total_q,
                    total_k, workspace, workspace_bytes, true, dtype, stream);
}

// ------------------------------------------------------------------ allocation-free backward
// Scratch for D = rowsum(dO ∘ O) when the caller cannot provide a workspace: a fixed array
// in this module's device memory (every GPU that loads the library holds it until exit).
constexpr size_t kNoAllocScratchFloats = size_t(1) << 22;  // 16 MiB: B*H*N <= 4194304
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// Device address of the scratch array on the current device, looked up once per device
// with that device current (the host-side symbol is only a stand-in and must never be
// handed to a kernel).
static int noalloc_scratch(float** out) {
  static PerDeviceSymbol<float> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev >= PerDeviceSymbol<float>::kMaxDevices) return fail(FA_ERR_UNSUPPORTED, "device index >= 64");
  float* p = cache.get(g_noalloc_scratch, dev, &e);
  if (p == nullptr) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
  *out = p;
  return FA_OK;
}

int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int N, int H, int d,
                   float scale, int causal, int dtype, void* stream) {
  g_last_error.clear();
  if (int e = check_common(H, d, dtype, scale)) return e;
  if (B < 0 || N < 0) return fail(FA_ERR_INVALID_ARG, "B and N must be >= 0");
  if ((long long)B * N >= (1LL << 31)) return fail(FA_ERR_UNSUPPORTED, "B*N must be < 2^31");
  if (B == 0 || N == 0 || H == 0) return FA_OK;
  if ((unsigned long long)B * H * N > kNoAllocScratchFloats)
    return fail(FA_ERR_UNSUPPORTED,
                "B*H*N = " + std::to_string((unsigned long long)B * H * N) +
                    " exceeds the allocation-free scratch capacity of " +
                    std::to_string(kNoAllocScratchFloats) + " (use fa_bwd with a workspace)");
  if (int e = check_grid(B, H, N)) return e;
  float* scratch = nullptr;
  if (int e = noalloc_scratch(&scratch)) return e;
  return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, nullptr, nullptr, H, d, scale, -1,
                    causal ? 0 : -1, (long long)B * N, (long long)B * N, N, B, N, N, B * N, B * N,
                    scratch, sizeof(float) * kNoAllocScratchFloats, false, dtype,
                    (cudaStream_t)stream);
}

// ------------------------------------------------------------------ KV-cache decode
namespace {

// Split policy: enough CTAs for about eight waves of 148 SMs, whole 128-key tiles per
// split.  A fixed function of (B, H, max_seqlen_k), so fa_decode_workspace_size can size
// the partial results without a device.
constexpr long long kDecodeTargetCtas = 8LL * 148;

void decode_splits(long long B, long long H, long long max_len, int* splits, int* chunk) {
  const long long tiles = max_len > 0 ? (max_len + 127) / 128 : 1;
  long long want = (kDecodeTargetCtas + B * H - 1) / (B * H);
  want = std::max(1LL, std::min(want, tiles));
  const long long per = (tiles + want - 1) / want;  // tiles per split
  *splits = (int)((tiles + per - 1) / per);
  *chunk = (int)(per * 128);
}

size_t decode_workspace(long long B, long long Nq, long long H, long long d, long long max_len) {
  int splits = 1, chunk = 128;
  decode_splits(B, H, max_len, &splits, &chunk);
  if (splits <= 1) return 0;
  const size_t rows = (size_t)B * Nq * H * splits;
  return align256(rows * d * 4) + align256(rows * 4);
}

int decode_common(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* block_table, const int* cache_seqlens, int B, int Nq, int H, int d,
                  long long cache_rows, long long cache_batches, int box_rows, int max_len,
                  int page_size, int max_blocks, int num_pages, float scale, int causal,
                  void* workspace, size_t workspace_bytes, int dtype, void* stream) {
  if (int e = check_ptrs({q, o, lse, cache_seqlens})) return e;
  if (int e = check_ptrs({k, v})) return e;
  if (block_table != nullptr)
    if (int e = check_ptrs({block_table})) return e;
  DecParams p{};
  p.q = q;
  p.o = o;
  p.lse = lse;
  p.seqlens = cache_seqlens;
  p.block_table = block_table;
  p.B = B;
  p.Nq = Nq;
  p.H = H;
  p.max_len = max_len;
  p.page_size = page_size;
  p.max_blocks = max_blocks;
  p.num_pages = num_pages;
  decode_splits(B, H, max_len, &p.splits, &p.chunk);
  const size_t need = decode_workspace(B, Nq, H, d, max_len);
  if (need > 0) {
    if (workspace == nullptr) return fail(FA_ERR_INVALID_ARG, "decode needs a workspace");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return fail(FA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (workspace_bytes < need)
      return fail(FA_ERR_INVALID_ARG, "workspace too small (need " + std::to_string(need) + " bytes)");
    const size_t rows = (size_t)B * Nq * H * p.splits;
    p.o_part = static_cast<float*>(workspace);
    p.lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align256(rows * d * 4));
  }
  p.scale_log2 = scale * kLog2e;
  p.win_left = -1;
  p.win_right = causal ? 0 : -1;
  p.status = status_ptr();
  if (p.status == nullptr) return cuda_fail(cudaGetLastError(), "status word");
  CUtensorMap mk, mv;
  if (int e = make_map(&mk, k, d, H, cache_rows, cache_batches, box_rows)) return e;
  if (int e = make_map(&mv, v, d, H, cache_rows, cache_batches, box_rows)) return e;
  return launch_result(launch_decode(d, dtype == FA_BF16, block_table != nullptr, mk, mv, p,
                                     (cudaStream_t)stream));
}

int decode_check(int B, int Nq, int H, int d, int max_seqlen_k, float scale, int dtype) {
  if (int e = check_common(H, d, dtype, scale)) return e;
  if (B < 0 || Nq < 0 || max_seqlen_k < 0) return fail(FA_ERR_INVALID_ARG, "sizes must be >= 0");
  if (Nq > kDecodeMaxQueries)
    return fail(FA_ERR_UNSUPPORTED, "decode takes at most " + std::to_string(kDecodeMaxQueries) +
                                        " query rows per sequence");
  if (B > 65535) return fail(FA_ERR_UNSUPPORTED, "B must be <= 65535");
  return FA_OK;
}

}  // namespace

size_t fa_decode_workspace_size(int B, int Nq, int H, int d, int max_seqlen_k) {
  if (B <= 0 || Nq <= 0 || H <= 0 || d <= 0 || max_seqlen_k < 0) return 0;
  return decode_workspace(B, Nq, H, d, max_seqlen_k);
}

int fa_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
              const int* cache_seqlens, int B, int Nq, int H, int d, int cache_capacity,
              int max_seqlen_k, float scale, int causal, void* workspace, size_t workspace_bytes,
              int dtype, void* stream) {
  g_last_error.clear();
  if (int e = decode_check(B, Nq, H, d, max_seqlen_k, scale, dtype)) return e;
  if (cache_capacity < 0) return fail(FA_ERR_INVALID_ARG, "cache_capacity must be >= 0");
  if (max_seqlen_k > cache_capacity)
    return fail(FA_ERR_INVALID_ARG, "max_seqlen_k exceeds cache_capacity");
  if (B == 0 || Nq == 0 || H == 0) return FA_OK;
  // An empty cache is never read; any aligned buffer stands in for the tensor map.
  const bool empty = cache_capacity == 0;
  return decode_common(q, empty ? q : k_cache, empty ? q : v_cache, o, lse, nullptr,
                       cache_seqlens, B, Nq, H, d, empty ? 1 : cache_capacity, empty ? 1 : B,
                       128, max_seqlen_k, 0, 0, 0, scale, causal, workspace, workspace_bytes,
                       dtype, stream);
}

int fa_decode_paged(const void* q, const void* k_pages, const void* v_pages, void* o, float* lse,
                    const int* block_table, const int* cache_seqlens, int B, int Nq, int H, int d,
                    int page_size, int num_pages, int max_blocks_per_seq, int max_seqlen_k,
                    float scale, int causal, void* workspace, size_t workspace_bytes, int dtype,
                    void* stream) {
  g_last_error.clear();
  if (int e = decode_check(B, Nq, H, d, max_seqlen_k, scale, dtype)) return e;
  if (page_size < 16 || (page_size & (page_size - 1)) != 0)
    return fail(FA_ERR_UNSUPPORTED, "page_size must be a power of two >= 16");
  if (num_pages <= 0 || max_blocks_per_seq <= 0)
    return fail(FA_ERR_INVALID_ARG, "num_pages and max_blocks_per_seq must be >= 1");
  if ((long long)max_blocks_per_seq * page_size < max_seqlen_k)
    return fail(FA_ERR_INVALID_ARG, "max_seqlen_k exceeds max_blocks_per_seq * page_size");
  if (B == 0 || Nq == 0 || H == 0) return FA_OK;
  if (block_table == nullptr) return fail(FA_ERR_INVALID_ARG, "null pointer argument");
  return decode_common(q, k_pages, v_pages, o, lse, block_table, cache_seqlens, B, Nq, H, d,
                       page_size, num_pages, std::min(page_size, 128), max_seqlen_k, page_size,
                       max_blocks_per_seq, num_pages, scale, causal, workspace, workspace_bytes,
                       dtype, stream);
}

int fa_get_device_status(void* stream) {
  g_last_error.clear();
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t* sp = status_ptr();
  if (sp == nullptr) return cuda_fail(cudaGetLastError(), "status word");
  uint32_t word = 0;
  e = cudaMemcpy(&word, sp, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read status word");
  if (word != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpy(sp, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clear status word");
    if (word & kDevTimeout) return fail(FA_ERR_TIMEOUT, "a kernel wait timed out");
    if (word & kDevBadSeqlens)
      return fail(FA_ERR_INVALID_ARG,
                  "a varlen call saw cu_seqlens outside [0, total] or a sequence longer than "
                  "max_seqlen (that sequence was skipped)");
    if (word & kDevBadCache)
      return fail(FA_ERR_INVALID_ARG,
                  "a decode call saw a cache length above its bounds or a page id out of range");
    if (word & kDevSmemAlign)
      return fail(FA_ERR_UNSUPPORTED, "dynamic shared memory base not 1024-byte alignable");
  }
  return FA_OK;
}

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

const char* fa_last_error(void) { return g_last_error.c_str(); }

int fa_selftest_exp2(const float* x, float* y, int n, void* stream) {
  g_last_error.clear();
  if (n < 0) return fail(FA_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return FA_OK;
  if (x == nullptr || y == nullptr) return fail(FA_ERR_INVALID_ARG, "null pointer argument");
  const int pairs = (n + 1) / 2;
  selftest_exp2_kernel<<<(pairs + 255) / 256, 256, 0, (cudaStream_t)stream>>>(x, y, n);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e, "selftest_exp2 launch");
}

int fa_selftest_fwd_f32(const void* q, const void* k, const void* v, float* o, float* lse, int B,
                        int N, int H, int d, float scale, int window_left, int window_right,
                        int dtype, void* stream) {
  g_last_error.clear();
  if (int e = check_common(H, d, dtype, scale)) return e;
  if (B < 0 || N < 0) return fail(FA_ERR_INVALID_ARG, "B and N must be >= 0");
  if ((long long)B * N >= (1LL << 31)) return fail(FA_ERR_UNSUPPORTED, "B*N must be < 2^31");
  if (B == 0 || N == 0 || H == 0) return FA_OK;
  if (int e = check_grid(B, H, N)) return e;
  int wl = window_left, wr = window_right;
  if (int e = normalize_window(&wl, &wr, N, N)) return e;
  if (int e = check_ptrs({q, k, v, o, lse})) return e;
  CUtensorMap mq, mk, mv;
  if (int e = make_map(&mq, q, d, H, N, B, 128)) return e;
  if (int e = make_map(&mk, k, d, H, N, B, 128)) return e;
  if (int e = make_map(&mv, v, d, H, N, B, 128)) return e;
  FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.N = N;
  p.H = H;
  p.total_q = B * N;
  p.scale = scale;
  set_fwd_scale(p, scale);
  p.win_left = wl;
  p.win_right = wr;
  p.reverse_tiles = reverse_tiles(wl, wr);
  p.max_seqlen_q = N;
  p.status = status_ptr();
  if (p.status == nullptr) return cuda_fail(cudaGetLastError(), "status word");
  const int rows = fwd_rows_per_cta(false);
  dim3 grid((N + rows - 1) / rows, H, B);
  return launch_result(
      launch_fwd_f32out(d, dtype == FA_BF16, mq, mk, mv, /*unused*/ mq, p, grid,
                        (cudaStream_t)stream));
}

int fa_selftest_wait_timeout(unsigned int limit_us, void* stream) {
  g_last_error.clear();
  uint32_t* sp = status_ptr();
  if (sp == nullptr) return cuda_fail(cudaGetLastError(), "status word");
  selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(sp, (uint64_t)limit_us * 1000ull);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return fa_get_device_status(stream);
}

}  // extern "C"
