/*
 * fattn — exact scaled-dot-product attention, tile by tile with online softmax, for
 * NVIDIA B200 (sm_100a).  Plain C ABI: device pointers, sizes, a CUDA stream handle.
 *
 * What is computed.  For every (batch, head) — or, for the varlen calls, every packed
 * sequence and head — with queries Q [Lq, d], keys K [Lk, d] and values V [Lk, d]:
 *
 *     S = scale · Q Kᵀ,   P = softmax(S) over keys,   O = P V,
 *     LSE_i = ln Σ_j exp(S_ij)          (natural log, scaled-score units)
 *
 * the "standard attention" of the page "FlashAttention-2的核心设计原理" (yunthe.com),
 * section "FlashAttention-2与标准注意力的计算对比", evaluated exactly but tile by tile
 * with a running row maximum and a rescaled running sum (page
 * "FlashAttention实战：如何在A100上实现3倍加速的Transformer训练" §3.1), so that the
 * N×N score matrix is never stored.  The backward calls recompute P from Q, K and the
 * saved LSE (page "Flash Attention V3：大模型训练加速与显存优化技术解析" §3.2).
 *
 * Causal masking (flag `causal`): key j is allowed for query i iff j <= i + (Lk - Lq)
 * (bottom-right alignment; the usual lower triangle when Lq == Lk).  A query row with no
 * allowed key gets O = 0, LSE = +inf and contributes nothing to any gradient.
 *
 * Layouts (all contiguous, head_dim innermost):
 *   dense  q, k, v, o, dout, dq, dk, dv : [B, N, H, d]   (the pages' [batch, seqlen,
 *          heads, head_dim], "FlashAttention-2的核心设计原理" section
 *          "FlashAttention-2反向传播与多GPU训练")
 *   dense  lse                         : [B, H, N] float32
 *   varlen q, o, dout, dq              : [total_q, H, d];  k, v, dk, dv : [total_k, H, d]
 *   varlen lse                         : [H, total_q] float32
 *   cu_seqlens_q / cu_seqlens_k        : device int32 [num_seqs + 1], cu[0] = 0,
 *          non-decreasing, cu[num_seqs] = total (section
 *          "变长序列处理与flash_attn_varlen_func" of the same page)
 * Element type of q/k/v/o/dout/dq/dk/dv: FA_BF16 or FA_FP16 (all the same); every MMA
 * accumulates in fp32; 16-bit results are rounded to nearest-even.
 * head_dim d must be 64 or 128.  Every device pointer must be 16-byte aligned.
 *
 * Ownership.  The caller allocates and owns every buffer.  The library allocates no
 * device memory at call time.  The backward calls take a caller-provided workspace sized
 * by fa_bwd_workspace_size / fa_varlen_bwd_workspace_size.  The library's module holds
 * two fixed device arrays on every GPU that loads it, until the process exits: one status
 * word (see fa_get_device_status) and the 16 MiB scratch array of fa_bwd_noalloc (held
 * even when fa_bwd_noalloc is never called).
 *
 * Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream):
 * they validate, launch and return.  Validation failures return a non-zero status,
 * launch nothing and leave every output untouched.  A device-side bounded wait that
 * runs out (a pipeline that stopped making progress) is reported later by
 * fa_get_device_status; the kernel then finishes without hanging the GPU and its
 * outputs are undefined.
 */
#ifndef FATTN_H_
#define FATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative size, bad cu_seqlens count;
                             from fa_get_device_status: a malformed cu_seqlens segment or
                             decode cache bounds exceeded on the device */
  FA_ERR_UNSUPPORTED = 2, /* head_dim other than 64/128, unknown dtype, size limits */
  FA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (see fa_last_error) */
  FA_ERR_TIMEOUT = 4      /* a kernel's bounded wait ran out (fa_get_device_status) */
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

/* Dense forward.  Writes o [B,N,H,d] and lse [B,H,N].
 * Sizes: B, N, H >= 0 (a zero size is a no-op), B*N < 2^31, H < 2^16,
 * B <= 65535.
 * scale: any finite float (the pages use 1/sqrt(d)). */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N,
           int H, int d, float scale, int causal, int dtype, void* stream);

/* Varlen forward over packed sequences (flash_attn_varlen_func semantics).
 * Writes o [total_q,H,d] and lse [H,total_q].
 * max_seqlen_q / max_seqlen_k must be >= every sequence's length; num_seqs, total_q,
 * total_k are the host-side counts matching cu_seqlens (the host cannot read device
 * cu_seqlens without a synchronisation).  num_seqs <= 65535.  Together they size the grid:
 * one CTA per 128-row tile of all sequences ((total + 127 num_seqs) / 128 at most) when
 * that is well below one slot per tile of the longest sequence for every sequence and
 * num_seqs <= 1024, otherwise the latter.
 * The kernels check every segment before using it: a segment outside [0, total_q) or
 * [0, total_k), or longer than max_seqlen_q (forward, dQ) or max_seqlen_k (dK/dV), is
 * skipped (its outputs are left unwritten) and fa_get_device_status then returns
 * FA_ERR_INVALID_ARG; nothing is accessed out of bounds. */
int fa_varlen_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int max_seqlen_q,
                  int max_seqlen_k, int H, int d, float scale, int causal, int num_seqs,
                  int total_q, int total_k, int dtype, void* stream);

/* Workspace bytes the dense backward needs: D = rowsum(dO ∘ O) [B,H,N] fp32 rounded up to
 * a multiple of 256 bytes, followed by the fp32 sums of dQ ([B,N,H,d], again rounded to 256
 * bytes).  Linear in N: no N x N buffer exists. */
size_t fa_bwd_workspace_size(int B, int N, int H, int d);

/* Dense backward: recomputes P from q, k and lse (as written by fa_fwd with the same
 * scale and causal flag) and writes dq, dk, dv [B,N,H,d].
 * One pass per 128-key tile computes the five products of every (query tile, key tile)
 * pair — Sᵀ = K Qᵀ, dPᵀ = V dOᵀ, dV += Pᵀ dO, dK += dSᵀ Q and dQ += dS K — ("global
 * gradients split into local updates", page "Flash Attention V3：大模型训练加速与显存优化
 * 技术解析" §3.2); the dQ contributions of the key tiles are added into the workspace's
 * fp32 sums with atomic adds, then rounded to 16 bits.  dK and dV are bitwise
 * reproducible; dQ may differ in its last bits from run to run (the order of the fp32
 * additions varies).  fa_bwd_deterministic gives bitwise-reproducible dQ as well.
 * o and dout are [B,N,H,d]; workspace must hold fa_bwd_workspace_size bytes and be
 * 256-byte aligned; its contents on entry do not matter. */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
           const float* lse, void* dq, void* dk, void* dv, int B, int N, int H, int d,
           float scale, int causal, void* workspace, size_t workspace_bytes, int dtype,
           void* stream);

/* Workspace bytes the varlen backward needs: D [H,total_q] fp32 and the fp32 dQ sums
 * ([total_q,H,d]), each rounded up to a multiple of 256 bytes. */
size_t fa_varlen_bwd_workspace_size(int total_q, int H, int d);

/* Varlen backward; arguments as fa_varlen_fwd plus the gradient buffers.  Computed as
 * fa_bwd (single pass, atomically added dQ). */
int fa_varlen_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                  const int* cu_seqlens_k, int max_seqlen_q, int max_seqlen_k, int H, int d,
                  float scale, int causal, int num_seqs, int total_q, int total_k,
                  void* workspace, size_t workspace_bytes, int dtype, void* stream);

/* Deterministic backward (the pages' deterministic=True mode, page
 * "FlashAttention实战：如何在A100上实现3倍加速的Transformer训练" §4.2): the same results as
 * fa_bwd / fa_varlen_bwd within rounding, bitwise reproducible from run to run.  Two
 * passes instead of one: dK and dV per key tile, then dQ per query tile (each recomputes S
 * and dP: seven products per tile pair instead of five), so that every gradient element is
 * written exactly once and no fp32 sum depends on timing.  The window arguments are those
 * of the _local calls ((-1, 0) causal, (-1, -1) full attention).  workspace: only its
 * first part (D, B*H*N or H*total_q floats rounded up to 256 bytes) is used; a workspace
 * sized by fa_bwd_workspace_size / fa_varlen_bwd_workspace_size is more than enough. */
int fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                         int N, int H, int d, float scale, int window_left, int window_right,
                         void* workspace, size_t workspace_bytes, int dtype, void* stream);

int fa_varlen_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                                const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                const int* cu_seqlens_q, const int* cu_seqlens_k,
                                int max_seqlen_q, int max_seqlen_k, int H, int d, float scale,
                                int window_left, int window_right, int num_seqs, int total_q,
                                int total_k, void* workspace, size_t workspace_bytes, int dtype,
                                void* stream);

/* ---------------------------------------------------------------- local attention
 * Sliding-window (local) attention: the variant listed by the page "FlashAttention技术
 * 深度解析" (pwwt.cn/news/595117) in its CUDA backend feature table and in its section on
 * local attention, which give no parameters.  Read here as a window around the same
 * bottom-right-aligned diagonal the causal mask uses: key j is allowed for query i iff
 *
 *     i + (Lk - Lq) - window_left  <=  j  <=  i + (Lk - Lq) + window_right,
 *
 * a negative bound meaning no bound on that side.  (-1, 0) is the causal mask, (-1, -1)
 * full attention, (w, 0) causal attention over the last w + 1 keys.  Key tiles that no
 * row of a query tile may see are skipped, so the work grows with the window, not with
 * the sequence.  Rows whose window holds no key behave like fully masked causal rows
 * (O = 0, LSE = +inf, no gradient contribution).  Bounds at or above the sequence
 * lengths are the same as no bound.  With any bound other than the causal one,
 * max_seqlen_q + max_seqlen_k (dense: 2N) must be < 2^31 (FA_ERR_UNSUPPORTED otherwise).
 * Every other argument, layout, limit and error is that of the call without _local. */
int fa_fwd_local(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N,
                 int H, int d, float scale, int window_left, int window_right, int dtype,
                 void* stream);

int fa_varlen_fwd_local(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int max_seqlen_q,
                        int max_seqlen_k, int H, int d, float scale, int window_left,
                        int window_right, int num_seqs, int total_q, int total_k, int dtype,
                        void* stream);

/* Backward of fa_fwd_local: lse must come from fa_fwd_local with the same scale and
 * window; workspace as for fa_bwd. */
int fa_bwd_local(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, int B, int N, int H, int d,
                 float scale, int window_left, int window_right, void* workspace,
                 size_t workspace_bytes, int dtype, void* stream);

int fa_varlen_bwd_local(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int max_seqlen_q,
                        int max_seqlen_k, int H, int d, float scale, int window_left,
                        int window_right, int num_seqs, int total_q, int total_k,
                        void* workspace, size_t workspace_bytes, int dtype, void* stream);

/* ---------------------------------------------------------------- FP8 forward
 * Forward pass with 8-bit inputs: the pages credit FP8 tensor-core support to Hopper and
 * quote FP8 attention at over 1.2 PFLOPS with an 8-bit quantization strategy (page
 * "FlashAttention实战：如何在A100上实现3倍加速的Transformer训练" §7, page "Flash
 * Attention V3：大模型训练加速与显存优化技术解析" §2.1) without fixing a format or scaling.
 * Read here as: q, k, v hold OCP FP8 E4M3 bytes, one dequantisation factor per tensor, and
 * the result is fa_fwd's O and LSE for the real inputs q_descale·Q8, k_descale·K8,
 * v_descale·V8 (layouts as fa_fwd / fa_varlen_fwd with 1-byte elements).
 * Both products run on the 8-bit tensor cores with fp32 accumulation; the softmax weights
 * P are themselves rounded to E4M3 (scaled into its normal range) for the P·V product and
 * O is normalised by the sum of the rounded weights, so O carries a relative error of at
 * most 2^-4/(1 - 2^-4) of sum_j P_ij |v_j - O_i| (per element) beyond the 16-bit output
 * rounding; LSE is computed from the unrounded weights (fa_fwd's accuracy).
 * d must be 128; scale finite and >= 0; descale factors finite and > 0.  o is written in
 * out_dtype (FA_BF16 or FA_FP16). */
int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N,
               int H, int d, float scale, float q_descale, float k_descale, float v_descale,
               int causal, int out_dtype, void* stream);

int fa_varlen_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                      const int* cu_seqlens_q, const int* cu_seqlens_k, int max_seqlen_q,
                      int max_seqlen_k, int H, int d, float scale, float q_descale,
                      float k_descale, float v_descale, int causal, int num_seqs, int total_q,
                      int total_k, int out_dtype, void* stream);

/* ---------------------------------------------------------------- KV-cache decode
 * One incremental-decoding step: Nq new query tokens per sequence (1 <= Nq <= 16) attend
 * to the keys and values that sequence has cached.  KV caches for incremental decoding
 * and paged KV caches are features the page "FlashAttention技术深度解析"
 * (pwwt.cn/news/595117) lists (CUDA backend feature table; sections on causal masking
 * with KV-cache updates and incremental decoding, and on KV-cache management) without an
 * interface.  Read here as: sequence b has cache_seqlens[b] cached rows (the new tokens'
 * own keys and values already appended), and query row r sits at position
 * cache_seqlens[b] - Nq + r, so `causal` uses the same bottom-right alignment as fa_fwd.
 * Computes O and LSE exactly as fa_fwd would over that sequence's cached rows; rows of
 * the cache at or past cache_seqlens[b] are never used (they may hold anything).
 *
 * Layouts: q, o [B, Nq, H, d]; lse [B, H, Nq] fp32; cache_seqlens device int32 [B].
 *   fa_decode:       k_cache, v_cache [B, cache_capacity, H, d]
 *   fa_decode_paged: k_pages, v_pages [num_pages, page_size, H, d]; block_table device
 *                    int32 [B, max_blocks_per_seq]: logical page i of sequence b
 *                    (rows i*page_size ..) is physical page block_table[b][i].
 *                    page_size: a power of two >= 16.
 * max_seqlen_k: host-side bound on every cache_seqlens[b] (<= cache_capacity, or
 * <= max_blocks_per_seq * page_size); it sizes the split of each sequence over CTAs.
 * A device length above its bound, or a page id outside [0, num_pages), cannot be seen
 * on the host: the kernel clamps the length (reads nothing out of bounds, an invalid page
 * reads as zeros) and fa_get_device_status then returns FA_ERR_INVALID_ARG.
 * workspace: fa_decode_workspace_size(B, Nq, H, d, max_seqlen_k) bytes, 256-byte aligned
 * (fp32 partial results of the splits); may be NULL when that size is 0.
 * The arithmetic runs on the CUDA cores: the step is bound by reading the cache from HBM.
 * Same dtype, alignment, stream and error conventions as fa_fwd. */
size_t fa_decode_workspace_size(int B, int Nq, int H, int d, int max_seqlen_k);

int fa_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
              const int* cache_seqlens, int B, int Nq, int H, int d, int cache_capacity,
              int max_seqlen_k, float scale, int causal, void* workspace,
              size_t workspace_bytes, int dtype, void* stream);

int fa_decode_paged(const void* q, const void* k_pages, const void* v_pages, void* o,
                    float* lse, const int* block_table, const int* cache_seqlens, int B, int Nq,
                    int H, int d, int page_size, int num_pages, int max_blocks_per_seq,
                    int max_seqlen_k, float scale, int causal, void* workspace,
                    size_t workspace_bytes, int dtype, void* stream);

/* Allocation-free dense backward (no counterpart on the source pages: an interface
 * addition).  Same arguments as fa_bwd without the workspace, and the results of
 * fa_bwd_deterministic with the causal window (bitwise): the D vector
 * lives in a fixed array inside the library's device memory (16 MiB, held by every GPU
 * that loads the library until the process exits).  For callers that cannot obtain
 * device memory at call time: hosts whose device memory belongs entirely to another
 * allocator, or latency-critical loops that cannot afford cudaMalloc's implicit
 * synchronisation.  Nothing is allocated: no cudaMalloc, cudaFree or allocating library
 * routine is called.
 *   Limit: B*H*N <= 4194304, else FA_ERR_UNSUPPORTED with a message naming the limit.
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *   with that device current; make that first call before any stream capture.
 *   All calls on a device share the one array, which keeps the last call's contents
 *   (nothing in it needs to start at zero: every value read is written earlier in the
 *   same call).  Calls that overlap on the GPU (different streams, or host threads
 *   without ordering) race on it: order them on one stream or with events. */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int N, int H, int d,
                   float scale, int causal, int dtype, void* stream);

/* Synchronises `stream`, reads and clears the library's status word of the current
 * device, and reports what its kernels recorded since the last call, in this order:
 *   FA_ERR_TIMEOUT      a kernel's bounded wait ran out (its outputs are undefined);
 *   FA_ERR_INVALID_ARG  a varlen call met a cu_seqlens segment outside [0, total] or
 *                       longer than max_seqlen (that segment was skipped), or a decode
 *                       call met a cache length above its bound or a page id out of range;
 *   FA_ERR_UNSUPPORTED  the dynamic shared memory base could not be 1024-byte aligned;
 *   FA_OK               nothing recorded.
 * FA_ERR_CUDA if the synchronisation or the status read itself failed; fa_last_error then
 * names the step. */
int fa_get_device_status(void* stream);

/* Static description of a status code. */
const char* fa_status_string(int status);

/* Detail of the most recent failure on the calling host thread ("" if none). */
const char* fa_last_error(void);

/* Runs a one-CTA kernel whose only wait can never complete, with the given bound in
 * microseconds; used to test the timeout path without any tensor-core or TMA work in
 * flight.  Returns the status fa_get_device_status reports afterwards (FA_ERR_TIMEOUT
 * when the bounded wait works). */
int fa_selftest_wait_timeout(unsigned int limit_us, void* stream);

/* Evaluates, on the GPU, the FMA-pipe 2^x the forward softmax uses for part of its
 * exponentials (Cody–Waite range reduction plus a fitted degree-3 polynomial; inputs below
 * -126 clamp to -126; relative error <= 1e-4 for x >= -125, results of order 1e-38 below):
 * y[i] = 2^x[i] for i < n, device pointers, asynchronous on `stream`.
 * A self-test hook with no counterpart on the pages. */
int fa_selftest_exp2(const float* x, float* y, int n, void* stream);

/* fa_fwd_local with O written in fp32 before it is rounded to 16 bits (o: float
 * [B,N,H,d]); lse as fa_fwd.  The same kernel as fa_fwd / fa_fwd_local in a test-only
 * instance, so that a parity test can hold the output to the accuracy target
 * |O - O_ref| <= 1e-2 (page "FlashAttention-2的核心设计原理", section
 * "FlashAttention-2与标准注意力的计算对比") where the 16-bit rounding of a large |O| alone can
 * exceed it.  Window (-1, 0) is causal, (-1, -1) full attention; other arguments and
 * conventions as fa_fwd_local; o must be 16-byte aligned. */
int fa_selftest_fwd_f32(const void* q, const void* k, const void* v, float* o, float* lse,
                        int B, int N, int H, int d, float scale, int window_left,
                        int window_right, int dtype, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FATTN_H_ */
