// Thin inline-PTX wrappers for the Blackwell (sm_100a) features the attention kernels
// use: mbarriers with bounded waits, TMA tile loads/stores, the tensor memory (TMEM)
// allocator, tcgen05.mma with shared-memory / tensor-memory operands, tcgen05.ld/st.
//
// Operand formats (instruction descriptor and shared-memory matrix descriptor bit
// fields) follow the PTX ISA's tcgen05 chapter; they are hardware formats, so any
// correct encoder has the same fields.  Everything here is written for this library.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fattn {

// ------------------------------------------------------------------ status word
// Error codes a kernel can leave in the device status word (see fa_get_device_status).
enum : uint32_t {
  kDevOk = 0u,
  kDevTimeout = 1u,
  kDevSmemAlign = 2u,
  kDevBadCache = 4u,    // decode: cache length above its bound or page id out of range
  kDevBadSeqlens = 8u,  // varlen: a segment outside [0, total) or longer than the grid
};

// Varlen segment bz read from device prefix sums, checked before any use: rows
// [cu_q[bz], cu_q[bz+1]) must lie in [0, total_q) and keys likewise in [0, total_k), and the
// segment may hold at most q_cover rows and k_cover keys (the caller's max_seqlen_q /
// max_seqlen_k; negative: not checked).  A bad segment is reported in the status word and
// its CTA does nothing, so a malformed cu_seqlens never leads to an out-of-bounds access.
__device__ __forceinline__ bool varlen_bounds_ok(const int* cu_q, const int* cu_k, int bz,
                                                 int total_q, int total_k, long long q_cover,
                                                 long long k_cover) {
  const int q0 = cu_q[bz], q1 = cu_q[bz + 1], k0 = cu_k[bz], k1 = cu_k[bz + 1];
  return 0 <= q0 && q0 <= q1 && q1 <= total_q && 0 <= k0 && k0 <= k1 && k1 <= total_k &&
         (q_cover < 0 || q1 - q0 <= q_cover) && (k_cover < 0 || k1 - k0 <= k_cover);
}
__device__ __forceinline__ bool varlen_segment_ok(const int* cu_q, const int* cu_k, int bz,
                                                  int total_q, int total_k, long long q_cover,
                                                  long long k_cover, uint32_t* status) {
  const bool ok = varlen_bounds_ok(cu_q, cu_k, bz, total_q, total_k, q_cover, k_cover);
  if (!ok && threadIdx.x == 0) atomicOr(status, kDevBadSeqlens);
  return ok;
}
// Every segment checked by one CTA (its threads stride over them): with the packed grid
// below a segment without tiles has no CTA of its own to report it.
__device__ __forceinline__ void varlen_check_all(const int* cu_q, const int* cu_k, int nseg,
                                                 int total_q, int total_k, long long q_cover,
                                                 long long k_cover, uint32_t* status) {
  for (int s = threadIdx.x; s < nseg; s += blockDim.x)
    if (!varlen_bounds_ok(cu_q, cu_k, s, total_q, total_k, q_cover, k_cover))
      atomicOr(status, kDevBadSeqlens);
}

// Packed grid of a varlen launch: x numbers the 128-row tiles of all segments one segment
// after another (ceil(L_s / 128) tiles for segment s, L_s = cu[s+1] - cu[s]), so no CTA is
// launched for the tiles a short segment lacks.  Each warp finds the segment holding tile t
// with a running prefix sum over cu[], 32 segments per step (lengths clamped to
// [0, total] here; the CTA checks its own segment afterwards).  Returns false when t lies
// past the last tile.  Called by whole warps.
__device__ __forceinline__ bool packed_tile_lookup(const int* cu, int nseg, int total, int t,
                                                   int* seg, int* tile) {
  const int lane = threadIdx.x & 31;
  long long base = 0;  // tiles of segments 0 .. s0-1
  for (int s0 = 0; s0 < nseg; s0 += 32) {
    const int s = s0 + lane;
    int n = 0;
    if (s < nseg) {
      const long long len = (long long)cu[s + 1] - cu[s];
      n = (int)((min(max(len, 0ll), (long long)total) + 127) >> 7);
    }
    int incl = n;  // inclusive prefix sum over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int step = __shfl_sync(0xffffffffu, incl, 31);
    if (t < base + step) {
      const int ls = __ffs(__ballot_sync(0xffffffffu, t < base + incl)) - 1;
      *seg = s0 + ls;
      *tile = (int)(t - base) - __shfl_sync(0xffffffffu, incl - n, ls);
      return true;
    }
    base += step;
  }
  return false;
}

// Upper bound on a single mbarrier wait, in nanoseconds of %globaltimer.  A wait that
// runs out records kDevTimeout and makes every later wait in the same CTA return at
// once, so a broken pipeline ends instead of hanging the GPU.
#ifndef FATTN_WAIT_LIMIT_NS
#define FATTN_WAIT_LIMIT_NS 2000000000ull
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t elect_one_lane() { return (threadIdx.x & 31u) == 0u; }

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// Raises the phase's expected transaction bytes without an arrival (the arrival comes later).
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0u;
}

// Bounded wait for the phase with the given parity to complete.
// `abort_flag` is a CTA-shared word: once any wait in the CTA has timed out, all
// later waits return false immediately.  Returns true when the phase completed.
__device__ __forceinline__ bool mbar_wait_limit(uint32_t bar, uint32_t parity,
                                                volatile uint32_t* abort_flag, uint32_t* status,
                                                uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0u) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1u;
        atomicOr(status, kDevTimeout);
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile uint32_t* abort_flag, uint32_t* status) {
  return mbar_wait_limit(bar, parity, abort_flag, status, FATTN_WAIT_LIMIT_NS);
}

// ------------------------------------------------------------------ programmatic dependent launch
// In a kernel launched with programmatic stream serialisation: wait until the preceding
// kernel in the stream has completed and its memory writes are visible (a no-op otherwise).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// In the preceding kernel: allow the dependent launch to begin before this one completes.
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ register reallocation
// Executed by every warp of a warpgroup.  The sum over warpgroups must stay within the
// registers the CTA was launched with (threads x registers per thread at launch).
template <uint32_t N>
__device__ __forceinline__ void regs_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Named barrier for `count` threads (a multiple of 32) of the CTA; ids 1..15.
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ------------------------------------------------------------------ proxies and fences
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 4-D tiled load of one box into shared memory; completion is signalled on `bar` as
// transaction bytes.  No cluster multicast: each CTA loads what it uses.
__device__ __forceinline__ void tma_load_4d(const CUtensorMap* map, uint32_t bar, uint32_t dst,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

// 4-D tiled store of one box from shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
// 4-D tiled reduce-add of one fp32 box from shared memory into global memory (elementwise
// atomic adds done by the TMA unit; bulk-group completion).  Elements outside the tensor's
// extent are skipped.
__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap* map, uint32_t src, int c0,
                                                  int c1, int c2, int c3) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%2, %3, %4, %5}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
// Wait until at most one of this thread's bulk groups is still reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ------------------------------------------------------------------ TMEM allocation
// Called by one whole warp.  Writes the base TMEM address to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// ------------------------------------------------------------------ descriptors
// Instruction descriptor for tcgen05.mma kind::f16 with fp32 accumulation.
//   bits 4-5: D format (1 = f32); 7-9: A format; 10-12: B format (0 = f16, 1 = bf16);
//   bit 15: A is MN-major; bit 16: B is MN-major; 17-22: N >> 3; 24-28: M >> 4.
__host__ __device__ constexpr uint32_t idesc_f16_f32acc(bool bf16, int M, int N, bool a_mn_major,
                                                         bool b_mn_major) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
         ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand.
//   bits 0-13: start address >> 4; 16-29: leading-dimension byte offset >> 4;
//   32-45: stride-dimension byte offset >> 4; 46-47: version (1 on sm_100);
//   49-51: base offset (0: atoms are 1024-byte aligned); 61-63: layout (2 = 128B swizzle).
// K-major operands: rows of 128 bytes, 8-row atoms `sbo` apart (LBO unused).
// MN-major operands: 64-element runs along M/N, runs `lbo` apart; 8 K-rows of 128 bytes
// form an atom and atoms are `sbo` apart.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}

// Descriptor with its start address advanced by `bytes` (a multiple of 16).  Shared
// addresses stay below 256 KB, so the 14-bit start-address field never carries: building
// a descriptor once and adding compile-time offsets keeps the single MMA-issuing thread
// at one instruction pair per MMA (rebuilding descriptors per MMA made issue, not the
// tensor core, the bottleneck).
__device__ __forceinline__ uint64_t sdesc_adv(uint64_t d, uint32_t bytes) {
  return d + (uint64_t)(bytes >> 4);
}

// ------------------------------------------------------------------ tcgen05.mma
// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same two products for 8-bit operands (.kind::f8f6f4; both operands E4M3 here, the
// instruction descriptor's format code 0).  K per instruction is 32 elements (32 bytes).
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on `bar` when every tcgen05 async operation this thread issued so far
// has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// ------------------------------------------------------------------ tcgen05.ld / st
// 32 lanes x 32 bits, repeated N times along columns: thread t of the warp gets row
// (lane base + t), N consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Registers written by tcgen05.ld are only valid after tcgen05.wait::ld; this empty asm
// ties each register to a point after the wait so the compiler cannot read it earlier.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// ------------------------------------------------------------------ math helpers
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Round two fp32 values to nearest-even 16-bit and pack them (lo = first).
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  if constexpr (BF16) {
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  } else {
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  }
  return r;
}

// Paired fp32 arithmetic (sm_100): two lanes of fp32 in one 64-bit register pair.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return make_float2(lo, hi);
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for two values at once on the FMA pipe (paired fp32), so that part of the softmax
// exponentials bypass the special-function unit.  Method: Cody–Waite range reduction,
// x = j + f with j = rint(x) obtained by the 1.5·2^23 shift (round to nearest) and
// f in [-0.5, 0.5]; 2^f by a degree-3 polynomial whose coefficients were fitted for this
// library (minimax relative error on [-0.5, 0.5] by the Remez exchange algorithm in
// exp2_poly_fit.py beside this file, rounded to float32; max relative error 7.5e-5); 2^j by
// adding j to the exponent field.  Inputs below -126 are
// clamped to -126; below about -125 results approach the denormal range (~1e-38) and lose
// relative accuracy, and they are never exactly 0: do not use it where an exact 0 is
// required (masked keys).
__device__ __forceinline__ float2 exp2_poly2(float a, float b) {
  a = fmaxf(a, -126.f);
  b = fmaxf(b, -126.f);
  const uint64_t x = f2_pack(a, b);
  const uint64_t t = f2_add(x, f2_pack(12582912.f, 12582912.f));   // 1.5·2^23 + j
  const uint64_t j = f2_add(t, f2_pack(-12582912.f, -12582912.f));  // j (exact)
  const uint64_t f = f2_fma(j, f2_pack(-1.f, -1.f), x);             // f = x - j
  uint64_t p = f2_fma(f2_pack(0.0551716685295105f, 0.0551716685295105f), f,
                      f2_pack(0.2426111251115799f, 0.2426111251115799f));
  p = f2_fma(p, f, f2_pack(0.6932609677314758f, 0.6932609677314758f));
  p = f2_fma(p, f, f2_pack(0.9999280571937561f, 0.9999280571937561f));
  const float2 pf = f2_unpack(p), tf = f2_unpack(t);
  // bits(2^f) + (j << 23): j sits in the low mantissa bits of t (t = 0x4B400000 + j)
  const uint32_t ea = (__float_as_uint(tf.x) - 0x4B400000u) << 23;
  const uint32_t eb = (__float_as_uint(tf.y) - 0x4B400000u) << 23;
  return make_float2(__uint_as_float(__float_as_uint(pf.x) + ea),
                     __uint_as_float(__float_as_uint(pf.y) + eb));
}

// Round two fp32 values to E4M3 (nearest-even, saturating at ±448) and pack them into 16
// bits, lo = first (lower byte).
__device__ __forceinline__ uint32_t pack2_e4m3(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return (uint32_t)r;
}
// The two E4M3 values of the low 16 bits back to fp32 (exact), lo = first.
__device__ __forceinline__ float2 unpack2_e4m3(uint32_t v) {
  uint32_t h2;
  const uint16_t b = (uint16_t)(v & 0xFFFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(b));
  float lo, hi;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h2));
  return make_float2(lo, hi);
}

// Unpack two 16-bit floats (lo = first) to fp32.
template <bool BF16>
__device__ __forceinline__ float2 unpack2(uint32_t v) {
  if constexpr (BF16) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
  } else {
    float lo, hi;
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "cvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(v));
    return make_float2(lo, hi);
  }
}

}  // namespace fattn
