// Internal parameter blocks and launcher declarations shared by the library's
// translation units (not part of the public C ABI in include/fattn.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fattn {

// Forward kernel parameters.  Dense problems have cu_q == nullptr and use B, N;
// varlen problems index sequences through cu_q / cu_k (device int32 prefix sums).
struct FwdParams {
  void* o;          // [B, N, H, D] or [total_q, H, D], 16-bit
  float* lse;       // [B, H, N] or [H, total_q], fp32, natural log
  const int* cu_q;  // varlen only
  const int* cu_k;  // varlen only
  int N;            // dense sequence length
  int H;
  int total_q;      // varlen: rows of q/o (row stride of lse)
  float scale;      // softmax scale
  float scale_log2; // |scale| * log2(e), > 0 (a tiny positive value when scale == 0)
  int negate_scores;// 1 when scale < 0: the S product negates Q
  int causal;
  uint32_t* status; // device status word
};

// Backward kernel parameters (see bwd_kernels.cuh).
struct BwdParams {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;   // as written by the forward pass
  void* dq;
  void* dk;
  void* dv;
  float* dvec;        // D = rowsum(dO ∘ O), same layout as lse (caller's workspace)
  const int* cu_q;
  const int* cu_k;
  int B, N, H;
  int total_q, total_k;
  float scale;
  float scale_log2;
  int causal;
  uint32_t* status;
};

enum class LaunchResult { kOk, kUnsupported, kCudaError };

// Forward launch for one problem.  Tensor maps are built by the caller (api.cu).
LaunchResult launch_fwd(int d, bool bf16, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                        const CUtensorMap& tmV, const FwdParams& p, dim3 grid,
                        cudaStream_t stream);

// Forward grid: x = query-tile pairs, y = heads, z = batch (dense) or sequences (varlen).
int fwd_rows_per_cta();

// Backward launch: D preprocess, dK/dV pass, dQ pass.  q_rows = B*N (dense) or total_q
// (varlen); batches = B (dense) or num_seqs (varlen).
LaunchResult launch_bwd(int d, bool bf16, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                        const CUtensorMap& tmV, const CUtensorMap& tmDO, const BwdParams& p,
                        long long q_rows, int max_seqlen_q, int max_seqlen_k, int batches,
                        cudaStream_t stream);

}  // namespace fattn
