// sm_100a building blocks written as inline PTX: mbarriers with bounded waits, TMA
// tile loads, tcgen05 (tensor memory allocation, MMA, commit, loads/stores) and the
// shared-memory / instruction descriptors the MMAs take.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sigattn {

constexpr int kStatusTimeout = 1;

// Limit of the waits that end a kernel after another wait gave up: the copies a CTA issued
// and the MMAs it committed always complete, so these waits never depend on the caller's
// limit (which a test may set very short) and give up only if the hardware is gone.
constexpr unsigned long long kDrainWaitNs = 4000000000ull;

// What a bounded wait needs: the device status word to record a timeout in, the
// limit in nanoseconds, and a CTA-wide abort flag in shared memory that lets the other
// roles of the CTA stop waiting once one of them gave up.
struct WaitCtx {
  int* status;
  unsigned long long limit_ns;
  volatile int* abort;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }
__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }

// Item of round k of a persistent CTA's walk over a work list sorted longest-first: the
// CTAs take the items of even rounds in order and those of odd rounds in reverse ("snake"
// order), which evens out the work per CTA better than a plain stride (single-cell batch:
// at most 84 tiles per CTA instead of 89, mean 80.9).  Increasing in k for every CTA.
__device__ __forceinline__ int snake_item(int k) {
  const int g = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  return k * g + ((k & 1) ? g - 1 - c : c);
}

// ------------------------------------------------------------------------------------
// mbarrier
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test: has the phase with the given parity of `bar` completed?
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with the given parity of `bar` has completed.  Gives up when
// *w.abort becomes nonzero (another role gave up) or after w.limit_ns: then records the
// timeout in *w.status, raises *w.abort and returns false.  Never traps.
// The limit is checked on the SM cycle counter (cheap to read), at two cycles per
// nanosecond: never shorter than limit_ns at clocks up to 2 GHz.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  const long long limit = static_cast<long long>(w.limit_ns) * 2;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort) return false;
    if (clock64() - t0 > limit) {
      atomicOr(w.status, kStatusTimeout);
      *w.abort = 1;
      return false;
    }
  }
}

// ------------------------------------------------------------------------------------
// named barriers among a subset of warps
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ------------------------------------------------------------------------------------
// TMA
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 4-D tiled load (x = innermost element coordinate, must be a multiple of 8 for bf16).
__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
      : "memory");
}

// 4-D tiled reduce-add shared -> global (element type and box from the tensor map; box
// rows past the tensor's extent are not written).  Tracked as a bulk async-group of the
// issuing thread: bulk_commit_group() after it, then bulk_wait_read_1() (all but the newest
// group have read their sources) before a shared source is rewritten, and bulk_wait_all()
// before the kernel ends.
__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap* map, const void* smem_src,
                                                  int x, int y, int z, int w) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%1, %2, %3, %4}], [%5];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(smem_src))
      : "memory");
}

// Tiled bulk store shared -> global through a tensor map (rows and columns past the
// tensor's extent are not written); same completion rules as tma_reduce_add_4d.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* smem_src, int x,
                                             int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group"
      " [%0, {%1, %2, %3, %4}], [%5];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(smem_src))
      : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until at most one committed bulk group of this thread is still reading its source.
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// Waits until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Makes this thread's generic-proxy writes to shared memory visible to the async proxy
// (tensor-core operands, bulk copies) once a later barrier orders them.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Untiled bulk copy global -> shared, completing on `bar` (both addresses 16-byte
// aligned, `bytes` a multiple of 16).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------------------------------
// tcgen05: tensor memory
// ------------------------------------------------------------------------------------
// Allocates `ncols` (power of two, >= 32) TMEM columns; the base address is written to
// *dst_smem.  Executed by one whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

#define SIGATTN_R8(i) "=r"(r[i + 0]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                      "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define SIGATTN_W8(i) "r"(r[i + 0]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                      "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// Thread t of the warp reads TMEM lane (taddr.lane + t), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : SIGATTN_R8(0), SIGATTN_R8(8), SIGATTN_R8(16), SIGATTN_R8(24)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : SIGATTN_R8(0), SIGATTN_R8(8)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
                   taddr),
               SIGATTN_W8(0)
               : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      SIGATTN_W8(0), SIGATTN_W8(8), SIGATTN_W8(16), SIGATTN_W8(24)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      SIGATTN_W8(0), SIGATTN_W8(8)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------------------------
// Descriptors
// ------------------------------------------------------------------------------------
// Shared-memory matrix descriptor for a 128-byte-swizzled tile (sm_100 format):
//   bits  0-13 start address >> 4, 16-29 leading byte offset >> 4,
//   bits 32-45 stride byte offset >> 4, bit 46 version = 1, bits 61-63 layout (2 = 128B).
// K-major: rows of 128 bytes (64 bf16 along K), 8-row groups SBO = 1024 bytes apart,
//   LBO unused (1).  MN-major: 128-byte rows hold 64 consecutive N elements, one row per
//   K index; 8-row K groups SBO = 1024 apart; 64-wide N chunks LBO apart.
// The descriptor is kept as two 32-bit halves, for issue loops that step the start
// address: lo = start >> 4 | (lbo >> 4) << 16, hi = sbo >> 4 | version | layout.  Adding
// n to lo moves the start address by 16 n bytes; shared-memory addresses stay below
// 256 KB, so the 14-bit start field never carries into the offset field.
__host__ __device__ constexpr uint32_t sw128_desc_hi(uint32_t sbo_bytes) {
  return ((sbo_bytes >> 4) & 0x3FFF) | (1u << 14) | (2u << 29);
}
__device__ __forceinline__ uint32_t sw128_desc_lo(uint32_t saddr, uint32_t lbo_bytes) {
  return ((saddr & 0x3FFFF) >> 4) | (((lbo_bytes >> 4) & 0x3FFF) << 16);
}

// MMAs with the descriptors given as (lo, hi) halves sharing one hi word, issued by a whole
// warp: every lane runs the issue loop with the same (warp-uniform) operands and one lane
// elected by elect.sync issues.  Issuing from uniform values is markedly cheaper than from
// one lane's registers (12 MMAs + commit: 408 instead of 686 cycles, measured on B200).
__device__ __forceinline__ void mma_ss_lh_w(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                            uint32_t hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b64 da, db;\n\t"
      "mov.b64 da, {%1, %3};\n\tmov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_ts_lh_w(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                            uint32_t b_hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b64 db;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One tile's MMAs and the commit after them under a single elect.sync (whole-warp issue,
// as above).  PV of one 128-key tile: 8 K-steps of 16 keys, A (P, bf16 pairs) from TMEM
// columns a + 64 (k / 4) + 8 (k % 4), B (V, MN-major) at descriptor lo + 128 k; the first
// step accumulates iff acc0 != 0, the others always.
__device__ __forceinline__ void mma_pv8_commit_w(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                                 uint32_t b_hi, uint32_t idesc, uint32_t acc0,
                                                 uint64_t* bar) {
#define SIGATTN_PV_STEP(OA, OB)                                   \
  "add.u32 ra, %1, " #OA ";\n\tadd.u32 rl, %2, " #OB ";\n\t"     \
  "mov.b64 db, {rl, %3};\n\t"                                    \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], db, %4, q;\n\t"
  asm volatile(
      "{\n\t.reg .pred p, q, e;\n\t.reg .b64 db;\n\t.reg .b32 ra, rl;\n\t"
      "setp.ne.b32 p, %5, 0;\n\tsetp.ne.b32 q, %7, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t"
      SIGATTN_PV_STEP(8, 128) SIGATTN_PV_STEP(16, 256) SIGATTN_PV_STEP(24, 384)
      SIGATTN_PV_STEP(64, 512) SIGATTN_PV_STEP(72, 640) SIGATTN_PV_STEP(80, 768)
      SIGATTN_PV_STEP(88, 896)
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(acc0), "r"(smem_u32(bar)), "r"(1u)
      : "memory");
#undef SIGATTN_PV_STEP
}

// S = Q K^T of one tile (overwriting D) and the commit after it: K-steps of 16 columns of
// the 128B-swizzled K-major operands at descriptor offsets 2 (k % 4) + 1024 (k / 4) (16-byte
// units: 32 bytes within a 64-column box, 16 KB between boxes); 4 steps for d = 64, 8 for
// d = 128.
template <int kSteps>
__device__ __forceinline__ void mma_s_commit_w(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo,
                                               uint32_t hi, uint32_t idesc, uint64_t* bar) {
  static_assert(kSteps == 4 || kSteps == 8, "d = 64 or 128");
#define SIGATTN_S_STEP(OFF)                                                     \
  "add.u32 la, %1, " #OFF ";\n\tadd.u32 lb, %2, " #OFF ";\n\t"                \
  "mov.b64 da, {la, %3};\n\tmov.b64 db, {lb, %3};\n\t"                         \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, q;\n\t"
#define SIGATTN_S_HEAD                                                           \
  "{\n\t.reg .pred p, q, e;\n\t.reg .b64 da, db;\n\t.reg .b32 la, lb;\n\t"        \
  "setp.ne.b32 p, %6, 1;\n\tsetp.ne.b32 q, %6, 0;\n\telect.sync _|e, 0xffffffff;\n\t" \
  "mov.b64 da, {%1, %3};\n\tmov.b64 db, {%2, %3};\n\t"                              \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, p;\n\t"                   \
  SIGATTN_S_STEP(2) SIGATTN_S_STEP(4) SIGATTN_S_STEP(6)
#define SIGATTN_S_TAIL \
  "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t}\n"
  if constexpr (kSteps == 4) {
    asm volatile(SIGATTN_S_HEAD SIGATTN_S_TAIL ::"r"(d_tmem), "r"(a_lo), "r"(b_lo), "r"(hi),
                 "r"(idesc), "r"(smem_u32(bar)), "r"(1u)
                 : "memory");
  } else {
    asm volatile(SIGATTN_S_HEAD SIGATTN_S_STEP(1024) SIGATTN_S_STEP(1026) SIGATTN_S_STEP(1028)
                     SIGATTN_S_STEP(1030) SIGATTN_S_TAIL ::"r"(d_tmem),
                 "r"(a_lo), "r"(b_lo), "r"(hi), "r"(idesc), "r"(smem_u32(bar)), "r"(1u)
                 : "memory");
  }
#undef SIGATTN_S_STEP
#undef SIGATTN_S_HEAD
#undef SIGATTN_S_TAIL
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> fp32, dense.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format (1 = bf16),
//   bit 15 A major (0 = K), bit 16 B major (1 = MN), bits 17-22 N >> 3, bits 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major,
                                                      bool a_mn_major = false) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// ------------------------------------------------------------------------------------
// Whole-warp forms of commit and wait (see mma_ss_lh_w)
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void mma_commit_w(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Bounded wait for a whole converged warp: every lane runs the same wait loop.  try_wait,
// the cycle counter and the abort flag are read by one instruction for the whole warp, so
// the lanes see the same values and leave the loop together; no lane-0 branch, shuffle or
// reconvergence sits on the issue path.
__device__ __forceinline__ bool mbar_wait_w(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, w));
}

// ------------------------------------------------------------------------------------
// Numerics
// ------------------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (sm_100): one instruction for two lanes of math, same per-element
// throughput as scalar FFMA but half the issue slots.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// a * b clamped to [0, 1] (NaN gives 0); the packed form has no saturation, so two scalar
// multiplies (FMA pipe)
__device__ __forceinline__ float2 mul2_sat(float2 a, float2 b) {
  float2 d;
  asm("mul.rn.sat.f32 %0, %2, %4;\n\tmul.rn.sat.f32 %1, %3, %5;"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// a + b clamped to [0, 1] (NaN gives 0), two scalar adds as mul2_sat
__device__ __forceinline__ float2 add2_sat(float2 a, float2 b) {
  float2 d;
  asm("add.rn.sat.f32 %0, %2, %4;\n\tadd.rn.sat.f32 %1, %3, %5;"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Packs two floats into bf16x2 (round to nearest even); `lo` lands in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ------------------------------------------------------------------------------------
// Sigmoid with small relative error over the whole range, at one MUFU op per element.
//
// With t = x log2(e), e = 2^(-|t|) = exp(-|x|) in (0, 1] and g = 1 / (1 + e) in [1/2, 1):
//   sigma(x) = g for x >= 0,   sigma(x) = e g for x < 0,   sigma'(x) = sigma (1 - sigma) = e g^2
// (for x < 0: 1 - sigma(x) = sigma(-x) = g; for x >= 0: 1 - sigma = e g).  No cancellation
// anywhere, so the relative error of sigma is that of g plus that of exp2 -- unlike
// 0.5 + 0.5 tanh(x / 2), whose hardware tanh loses every digit of a weight like 1/n for
// long sequences (x = -log n well below -8).  e is the hardware exp2 (MUFU); g is the
// degree-4 polynomial below on the FMA pipe, fitted for minimal maximum relative error on
// [0, 1] (fit_sigmoid_poly.py): relative error 3.0e-4 = 2^-11.7 in float32, far below the
// bf16 rounding (2^-9) of the weights fed to the MMAs.
// A masked element takes t = -inf: e = 0, so sigma = sigma' = 0 there.
// ------------------------------------------------------------------------------------
constexpr float kSigG0 = 0.999702513f;
constexpr float kSigG1 = -0.984833419f;
constexpr float kSigG2 = 0.865889132f;
constexpr float kSigG3 = -0.532853127f;
constexpr float kSigG4 = 0.152243674f;

// e = 2^(-|t|) and g = 1 / (1 + e) for two elements.
__device__ __forceinline__ void sigmoid_parts2(float2 t, float2& e, float2& g) {
  e = make_float2(ex2_approx(-fabsf(t.x)), ex2_approx(-fabsf(t.y)));
  float2 a = fma2(make_float2(kSigG4, kSigG4), e, make_float2(kSigG3, kSigG3));
  a = fma2(a, e, make_float2(kSigG2, kSigG2));
  a = fma2(a, e, make_float2(kSigG1, kSigG1));
  g = fma2(a, e, make_float2(kSigG0, kSigG0));
}

// sigma from t, e and g without a compare-and-select (which would load the ALU pipe, the
// busiest pipe of the sigmoid epilogues): sigma = g m with m = 1 for x >= 0 and m = e for
// x < 0.  c = saturate(t 2^126) is 0 for t <= 0 and 1 for t > 2^-126 (values in between
// occur only where e rounds to 1), so m = saturate(e + c): three FMA-pipe operations.
__device__ __forceinline__ float2 sigmoid_select2(float2 t, float2 e, float2 g) {
  const float2 c = mul2_sat(t, make_float2(0x1p126f, 0x1p126f));
  return mul2(g, add2_sat(e, c));
}

// sigma(x) for two elements given t = x log2(e) (t = -inf for a masked element: 0).
__device__ __forceinline__ float2 sigmoid2(float2 t) {
  float2 e, g;
  sigmoid_parts2(t, e, g);
  return sigmoid_select2(t, e, g);
}

// sigma(x) and sigma'(x) = sigma (1 - sigma) = e g^2 for two elements, t as in sigmoid2.
__device__ __forceinline__ void sigmoid_grad2(float2 t, float2& p, float2& dp) {
  float2 e, g;
  sigmoid_parts2(t, e, g);
  p = sigmoid_select2(t, e, g);
  dp = mul2(mul2(e, g), g);
}

}  // namespace sigattn
