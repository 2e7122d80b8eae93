// Device helpers shared by the CSA2 kernels: error word, bounded mbarrier
// waits, TMA loads, tcgen05 (TMEM alloc, FP8 MMA, commit, load) and the shared
// memory / instruction descriptors of the sm_100a tensor cores.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

// ------------------------------------------------------------ constants ----
constexpr int kIndexHeads = CSA2_INDEX_HEADS;   // 32
constexpr int kIndexDim = CSA2_INDEX_DIM;       // 128 (FP8: 128 bytes per row)
constexpr int kKvDim = CSA2_KV_DIM;             // 512
constexpr int kKvCodeBytes = CSA2_KV_CODE_BYTES;
constexpr int kKvScaleBytes = CSA2_KV_SCALE_BYTES;
constexpr int kBlock = CSA2_BLOCK;              // positions per pool block
constexpr int kTile = 128;                      // positions per MMA tile (M)
constexpr int kPoolHistBins = CSA2_POOL_HIST_BINS;   // 4096: leading 12 bits of a block-max order key
constexpr int kPoolHistBits = 12;
static_assert(kPoolHistBins == 1 << kPoolHistBits, "one bin per leading-bit pattern");

// kernel ids recorded in err_word[1]
enum KernelId { kKAppend = 1, kKIndexFull = 2, kKPoolSelect = 3, kKReindex = 4, kKAttn = 5, kKPrefill = 6 };

// Wait bound of the pipeline barriers (ns of %globaltimer).  Well above any
// legitimate wait; a wait that runs out records CSA2_ERR_TIMEOUT and the CTA
// leaves its loops.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ void report_error(int32_t* err, int code, int kernel, int b, int idx) {
  if (err != nullptr && atomicCAS(err, 0, code) == 0) {
    err[1] = kernel;
    err[2] = b;
    err[3] = idx;
  }
}

// Visible positions of request b, or -1 for a length outside [0, capacity]
// (a corrupt ctx_len), which the caller that passes `report` records as
// CSA2_ERR_DEVICE_BOUNDS with the length as the index.  Callers treat such a
// request as empty: its results are left unwritten or padded, never computed
// over a truncated context, and none of its entries is checked or reported.
__device__ __forceinline__ int checked_ctx_len(const csa2_cache& c, int b, long long capacity, int kernel,
                                               bool report) {
  const int n = c.ctx_len[b];
  if (n < 0 || n > capacity) {
    if (report) report_error(c.err_word, CSA2_ERR_DEVICE_BOUNDS, kernel, b, n);
    return -1;
  }
  return n;
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Order-preserving map of an fp32 score to uint32 (larger score -> larger
// key); 0 is reserved for "not a candidate".
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  uint32_t k = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return k == 0u ? 1u : k;
}

// ------------------------------------------------------------- mbarrier ----
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of `parity` to complete, giving up after `limit_ns`.
// Returns false on time-out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > limit_ns) return false;
  }
}

// The same wait with a sleeping back-off between polls (32 ns doubling to
// 128 ns).  Every poll is a shared-memory operation; many warps polling at
// once take shared-memory bandwidth from the tensor cores' operand reads, so
// waits that are expected to last (an epilogue waiting for the next
// accumulator) use this form.
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  uint32_t ns = 32;
  while (true) {
    __nanosleep(ns);
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > limit_ns) return false;
    if (ns < 128) ns <<= 1;
  }
}

// Warp-uniform wait: lane 0 polls, the outcome is broadcast, so the whole warp
// leaves together (the tcgen05 loads that follow need a converged warp).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, limit_ns);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}
// Warp-uniform form of mbar_wait_backoff.
__device__ __forceinline__ bool mbar_wait_warp_backoff(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait_backoff(bar, parity, limit_ns);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}
// Warp-uniform read of a shared flag.
__device__ __forceinline__ bool warp_flag(const volatile int* flag) {
  int v = 0;
  if ((threadIdx.x & 31) == 0) v = *flag;
  return __shfl_sync(0xffffffffu, v, 0) != 0;
}

// ------------------------------------------- programmatic dependent launch ----
// A kernel launched with programmatic stream serialization may start while
// its predecessor in the stream is still running: it must call pdl_wait()
// before reading anything the predecessor writes.  pdl_launch_dependents()
// lets the next kernel in the stream be launched early.  Both are no-ops
// without a programmatic dependency.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------- named barriers ----
// bar.sync on barrier `id` (1..15) for `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// The same barrier, returning to every participant whether any of them passed
// a true predicate.
__device__ __forceinline__ bool named_bar_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// ------------------------------------------------------------------ TMA ----
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}
// 2-D tiled load (no multicast) into this CTA's shared memory; completion is
// signalled on `bar` as transaction bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}
// 1-D bulk copy global -> this CTA's shared memory (no multicast); both
// addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                             uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}
// Make generic-proxy writes to shared memory visible to the async proxy
// (tensor-core operand reads, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// -------------------------------------------------------------- tcgen05 ----
// TMEM allocation: executed by one full warp; the base address is written to
// shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, FP8 operands, fp32 accumulator.
__device__ __forceinline__ void umma_f8f6f4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// lane (warp quarter * 32 + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major operand stored as rows of 128
// bytes with the 128-byte swizzle (16-byte chunk c of row r lives at chunk
// c ^ (r % 8)); 8-row groups are 1024 bytes apart.  The base must be 1024-byte
// aligned; advancing along K inside the 128-byte row adds bytes/16 to the
// start-address field.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);   // start address
  d |= static_cast<uint64_t>(1) << 16;                        // LBO (unused here)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;                // SBO: 8 rows x 128 B
  d |= static_cast<uint64_t>(1) << 46;                        // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                        // 128-byte swizzle
  return d;
}

// Shared-memory matrix descriptor of a K-major operand stored as rows of 64
// bytes with the 64-byte swizzle (16-byte chunk c of row r lives at chunk
// c ^ ((r / 2) % 4)); 8-row groups are 512 bytes apart.  The base must be
// 512-byte aligned; a 32-byte step along K adds 2 to the start-address field.
__device__ __forceinline__ uint64_t sw64_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);   // start address
  d |= static_cast<uint64_t>(1) << 16;                        // LBO (unused here)
  d |= static_cast<uint64_t>(512 >> 4) << 32;                 // SBO: 8 rows x 64 B
  d |= static_cast<uint64_t>(1) << 46;                        // descriptor version
  d |= static_cast<uint64_t>(4) << 61;                        // 64-byte swizzle
  return d;
}
// Byte offset of (row, byte c) in a 64-byte-swizzled tile of 64-byte rows.
__host__ __device__ __forceinline__ uint32_t sw64_offset(uint32_t row, uint32_t c) {
  return row * 64u + ((((c >> 4) ^ (row >> 1)) & 3u) << 4) + (c & 15u);
}
// Descriptor of 32 rows x 16 bytes stored contiguously (the block-scale
// layout below) for tcgen05.cp: 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t scale_rows_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(128 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// Block scales of FP4 operands, in the order the tensor core reads them.  For
// a tile of 128 rows and 8 groups of 16 elements (K = 128) they take 1 KB:
// byte (g / 4) * 512 + (m % 32) * 16 + (m / 32) * 4 + g % 4 holds the scale of
// row m, group g.  Each 512-byte half (one K = 64 MMA) is 32 lines of 16 bytes,
// copied to tensor memory by one tcgen05.cp 32x128b.warpx4 (lines to lanes
// 0..31, replicated in the four lane quarters); the MMA then reads the scales
// of row m from lane m, column m / 32 of the copy.  An operand of N <= 128 rows
// (the query heads) uses the same layout.
__host__ __device__ constexpr uint32_t block_scale_offset(uint32_t m, uint32_t g) {
  return (g >> 2) * 512u + (m & 31u) * 16u + (m >> 5) * 4u + (g & 3u);
}

// tcgen05.cp of 32 lines x 16 bytes from shared memory to tensor memory
// columns taddr .. taddr + 3 of all four lane quarters.
__device__ __forceinline__ void tmem_cp_scales(uint32_t taddr, uint32_t smem_addr) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(scale_rows_desc(smem_addr))
               : "memory");
}

// D[tmem] (+)= (A * scale_A) x (B * scale_B)^T for FP4 (E2M1) operands with
// one E4M3 scale per 16 elements along K (K = 64 per instruction), fp32 D.
__device__ __forceinline__ void umma_mxf4nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor of kind::mxf4nvf4: A = B = E2M1, E4M3 block scales,
// fp32 D, both K-major, shape M x N, K = 64.
__host__ __device__ constexpr uint32_t idesc_mxf4nvf4(int M, int N) {
  return (1u << 7) | (1u << 10)                       // A, B: E2M1
         | (static_cast<uint32_t>(N >> 3) << 17)      // N / 8
         | (0u << 23)                                 // scales: E4M3
         | (static_cast<uint32_t>(M >> 4) << 24);     // M / 16
}

// Instruction descriptor of kind::f8f6f4: A = B = E4M3, D = fp32, both
// K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4)                                   // D format fp32
         | (0u << 7) | (0u << 10)                    // A, B: E4M3
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// ------------------------------------------------------- FP8 conversion ----
// Two fp32 -> two E4M3 bytes (round to nearest even, saturating); byte 0 of
// the result is `lo`.  -0 results are stored as +0.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  uint32_t v = r;
  if ((v & 0x007Fu) == 0) v &= 0xFF00u;
  if ((v & 0x7F00u) == 0) v &= 0x00FFu;
  return v;
}

// Smallest integer e >= -126 with 448 * 2^e >= amax (amax >= 0, finite).
// 448 = 1.75 * 2^8, so for amax = 1.m * 2^(E-127): e = E - 135 when
// 1.m <= 1.75 and E - 134 otherwise.
__device__ __forceinline__ int indexer_exponent(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int E = static_cast<int>(bits >> 23);
  int e = (E == 0) ? -126 : (((bits & 0x7FFFFFu) <= 0x600000u) ? E - 135 : E - 134);
  return e < -126 ? -126 : e;
}
// 2^k for k in [-126, 127] as an exact fp32.
__device__ __forceinline__ float exp2i(int k) { return __uint_as_float(static_cast<uint32_t>(k + 127) << 23); }

}  // namespace csa2
