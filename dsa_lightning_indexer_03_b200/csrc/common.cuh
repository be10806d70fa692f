// common.cuh -- sm_100a building blocks written for this library: mbarriers,
// TMA tile loads, tcgen05 (UMMA / TMEM) wrappers, bounded waits, and the
// order-preserving float <-> uint32 key used by the top-k selection.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dsa {

// ---------------------------------------------------------------- device error word bits
enum : int {
  kErrBounds = 1,    // a position / offset outside its sequence's cache rows
  kErrTimeout = 2,   // a bounded pipeline wait ran out; the kernel left early
  kErrOffsets = 4,   // malformed q_seq_offsets / cache_offsets
};

// ---------------------------------------------------------------- indexer constants
constexpr int kHeads = 32;      // indexer heads
constexpr int kHeadDim = 128;   // head dim == key dim
constexpr int kTopK = 2048;     // tokens kept per query
constexpr int kKeyTile = 128;   // keys per MMA tile (UMMA M)

// ---------------------------------------------------------------- small helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// barrier over `nthreads` threads that also ORs a predicate across them
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// float -> uint32 key whose unsigned order is the float order (-0 just below +0)
__device__ __forceinline__ uint32_t float_to_ordered(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ordered_to_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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
  return ok != 0;
}

// As mbar_try_wait, but the thread may stay suspended in hardware (up to
// kSuspendNs) until the phase completes instead of returning at once, so that a
// waiting warp does not take issue slots from the working ones.
constexpr uint32_t kSuspendNs = 20000;
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase.  Returns false (and raises the CTA's
// abort flag and the device error word) if the phase did not complete within
// timeout_ns, or if another role of the CTA already aborted.
struct WaitCtl {
  int* err;                 // device error word
  volatile int* abort_flag; // shared-memory flag, one per CTA
  uint64_t timeout_ns;
};

// the CTA's abort flag, read with an explicit shared-memory volatile load
__device__ __forceinline__ int read_abort(const WaitCtl& c) {
  int v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(const_cast<int*>(c.abort_flag))) : "memory");
  return v;
}

// bar is the barrier's shared-memory address.  A phase that has already completed is taken
// with one plain try_wait: the suspend-hinted form costs about 200 cycles even then.
__device__ __forceinline__ bool mbar_wait_addr(uint32_t a, uint32_t parity, const WaitCtl& c) {
  if (mbar_try_wait(a, parity)) return true;
  if (mbar_try_wait_sleep(a, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_sleep(a, parity)) return true;
    if (read_abort(c)) return false;
    if (global_timer_ns() - t0 > c.timeout_ns) {
      atomicOr(c.err, kErrTimeout);
      *c.abort_flag = 1;
      return false;
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtl& c) {
  return mbar_wait_addr(smem_u32(bar), parity, c);
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled load (no multicast) of the box at (x = inner coordinate, y = row)
// into shared memory; completion is signalled on `bar` as transaction bytes.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* m, uint64_t* bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// L2 eviction-priority policies for TMA loads (cache hints only; never affect results)
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 8-byte global store with an L2 cache policy.
__device__ __forceinline__ void st_global_u2_hint(uint2* p, uint2 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v2.u32 [%0], {%1, %2}, %3;" ::"l"(p), "r"(v.x), "r"(v.y), "l"(pol) : "memory");
}

// 2-D tiled load as tma_load_2d, with an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_hint(void* smem_dst, const CUtensorMap* m, uint64_t* bar, int32_t x,
                                                 int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// ---------------------------------------------------------------- tcgen05 (UMMA + TMEM)
// Shared-memory matrix descriptor of a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 64 bf16 (128 B), 8-row core groups 1024 B
// apart.  Fields: start address >> 4 (bits 0-13), leading-byte offset >> 4
// (16-29, unused for swizzled K-major, set to 1), stride-byte offset >> 4
// (32-45) = 1024 B, descriptor version 1 (bits 46-47), layout 2 = 128-byte
// swizzle (bits 61-63).  The tile base must be 1024-byte aligned; a K step of
// 16 elements inside the 128-byte row advances the start address by 32 B.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
  return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor of kind::f16 with bf16 A/B, fp32 accumulator, both
// operands K-major: D format (bits 4-5) = 1 (f32), A format (7-9) = 1 (bf16),
// B format (10-12) = 1 (bf16), N >> 3 (17-22), M >> 4 (24-28).
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor of kind::f8f6f4 with FP8 e4m3 A and B (format code 0 in both
// fields), fp32 accumulator, both operands K-major.
__host__ __device__ constexpr uint32_t umma_idesc_e4m3(int M, int N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
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

// D[tmem] (+)= A[smem] * B[smem]^T, one elected thread issues.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One 128-key tile: D[tmem] = sum over the 128-deep contraction of A (K-major SW128 tile of
// two 64-column halves, `a_half` bytes apart) times B (likewise, `b_half` apart), as 8
// tcgen05.mma of K = 16, the first overwriting D; then commits to both barriers.  The
// descriptors are formed from the low words of the two base descriptors (their address
// fields never carry: shared-memory addresses stay below 2^18).
template <uint32_t A_HALF, uint32_t B_HALF>
__device__ __forceinline__ void umma_tile_k128(uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr, uint32_t idesc,
                                               uint64_t* bar0, uint64_t* bar1) {
  const uint64_t ad = umma_desc_sw128(a_addr), bd = umma_desc_sw128(b_addr);
  const uint32_t alo = static_cast<uint32_t>(ad), ahi = static_cast<uint32_t>(ad >> 32);
  const uint32_t blo = static_cast<uint32_t>(bd), bhi = static_cast<uint32_t>(bd >> 32);
  asm volatile(
      "{\n\t.reg .pred p0, p1;\n\t.reg .b32 al, bl;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p0, %6, %6;\n\t"
      "setp.eq.b32 p1, %6, %6;\n\t"
      "mov.b64 a, {%1, %2};\n\tmov.b64 b, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, p0;\n\t"
      "add.u32 al, %1, 2;\n\tadd.u32 bl, %3, 2;\n\tmov.b64 a, {al, %2};\n\tmov.b64 b, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, p1;\n\t"
      "add.u32 al, %1, 4;\n\tadd.u32 bl, %3, 4;\n\tmov.b64 a, {al, %2};\n\tmov.b64 b, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, p1;\n\t"
      "add.u32 al, %1, 6;\n\tadd.u32 bl, %3, 6;\n\tmov.b64 a, {al, %2};\n\tmov.b64 b, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, p1;\n\t"
      "add.u32 al, %1, %7;\n\tadd.u32 bl, %3, %8;\n\tmov.b64 a, {al, %2};\n\tmov.b64 b, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, p1;\n\t"
      "add.u32 al, %1, %7+2;\n\tadd.u32 bl, %3, %8+2;\n\tmov.b64 a, {al, %2};\n\tmov.b64 b, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, p1;\n\t"
      "add.u32 al, %1, %7+4;\n\tadd.u32 bl, %3, %8+4;\n\tmov.b64 a, {al, %2};\n\tmov.b64 b, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, p1;\n\t"
      "add.u32 al, %1, %7+6;\n\tadd.u32 bl, %3, %8+6;\n\tmov.b64 a, {al, %2};\n\tmov.b64 b, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %5, p1;\n\t"
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%9];\n\t"
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%10];\n\t}"
      ::"r"(d_tmem), "r"(alo), "r"(ahi), "r"(blo), "r"(bhi), "r"(idesc), "r"(0), "n"(A_HALF >> 4), "n"(B_HALF >> 4),
      "r"(smem_u32(bar0)), "r"(smem_u32(bar1))
      : "memory");
}

// One 128-key tile of FP8 e4m3 operands: each 128-dim row is one 128-byte swizzle row, so the
// contraction is 4 tcgen05.mma.kind::f8f6f4 of K = 32 (32 bytes each), the first overwriting
// D; then commits to both barriers.
__device__ __forceinline__ void umma_tile_k128_e4m3(uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr,
                                                    uint32_t idesc, uint64_t* bar0, uint64_t* bar1) {
  const uint64_t ad = umma_desc_sw128(a_addr), bd = umma_desc_sw128(b_addr);
  const uint32_t alo = static_cast<uint32_t>(ad), ahi = static_cast<uint32_t>(ad >> 32);
  const uint32_t blo = static_cast<uint32_t>(bd), bhi = static_cast<uint32_t>(bd >> 32);
  asm volatile(
      "{\n\t.reg .pred p0, p1;\n\t.reg .b32 al, bl;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 p0, %6, %6;\n\t"
      "setp.eq.b32 p1, %6, %6;\n\t"
      "mov.b64 a, {%1, %2};\n\tmov.b64 b, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %5, p0;\n\t"
      "add.u32 al, %1, 2;\n\tadd.u32 bl, %3, 2;\n\tmov.b64 a, {al, %2};\n\tmov.b64 b, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %5, p1;\n\t"
      "add.u32 al, %1, 4;\n\tadd.u32 bl, %3, 4;\n\tmov.b64 a, {al, %2};\n\tmov.b64 b, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %5, p1;\n\t"
      "add.u32 al, %1, 6;\n\tadd.u32 bl, %3, 6;\n\tmov.b64 a, {al, %2};\n\tmov.b64 b, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %5, p1;\n\t"
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%7];\n\t"
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%8];\n\t}"
      ::"r"(d_tmem), "r"(alo), "r"(ahi), "r"(blo), "r"(bhi), "r"(idesc), "r"(0), "r"(smem_u32(bar0)),
      "r"(smem_u32(bar1))
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread i of the warp receives
// columns [col, col+32) of TMEM lane (lane base + i).
__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Packed fp32 pair FMA (sm_100): d = a * b + c elementwise on two lanes.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Waits for this thread's outstanding tcgen05.ld; the registers are passed
// through so the compiler cannot read them before the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
        "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]),
        "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
        "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

// tcgen05.ld 16x256b, x4: 16 TMEM lanes x 32 columns as four 8-column blocks.  Thread t
// receives, for block b, r[4b], r[4b+1] = (lane base + t/4, columns 8b + 2(t%4) + {0,1})
// and r[4b+2], r[4b+3] = the same columns of lane base + t/4 + 8.
// Four 16x256b.x4 loads (lane bases a0..a3) and the wait for them in one statement: the 64
// results are defined only after tcgen05.wait::ld.
__device__ __forceinline__ void tmem_ld4_16x256b_x4_wait(uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                         uint32_t (&r)[4][16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%65];\n\t"
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47}, [%66];\n\t"
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%67];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[0][4]), "=r"(r[0][5]), "=r"(r[0][6]),
        "=r"(r[0][7]), "=r"(r[0][8]), "=r"(r[0][9]), "=r"(r[0][10]), "=r"(r[0][11]), "=r"(r[0][12]),
        "=r"(r[0][13]), "=r"(r[0][14]), "=r"(r[0][15]),
        "=r"(r[1][0]), "=r"(r[1][1]), "=r"(r[1][2]), "=r"(r[1][3]), "=r"(r[1][4]), "=r"(r[1][5]), "=r"(r[1][6]),
        "=r"(r[1][7]), "=r"(r[1][8]), "=r"(r[1][9]), "=r"(r[1][10]), "=r"(r[1][11]), "=r"(r[1][12]),
        "=r"(r[1][13]), "=r"(r[1][14]), "=r"(r[1][15]),
        "=r"(r[2][0]), "=r"(r[2][1]), "=r"(r[2][2]), "=r"(r[2][3]), "=r"(r[2][4]), "=r"(r[2][5]), "=r"(r[2][6]),
        "=r"(r[2][7]), "=r"(r[2][8]), "=r"(r[2][9]), "=r"(r[2][10]), "=r"(r[2][11]), "=r"(r[2][12]),
        "=r"(r[2][13]), "=r"(r[2][14]), "=r"(r[2][15]),
        "=r"(r[3][0]), "=r"(r[3][1]), "=r"(r[3][2]), "=r"(r[3][3]), "=r"(r[3][4]), "=r"(r[3][5]), "=r"(r[3][6]),
        "=r"(r[3][7]), "=r"(r[3][8]), "=r"(r[3][9]), "=r"(r[3][10]), "=r"(r[3][11]), "=r"(r[3][12]),
        "=r"(r[3][13]), "=r"(r[3][14]), "=r"(r[3][15])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3)
      : "memory");
}

// Two 16x256b.x4 loads and their wait in one statement.
__device__ __forceinline__ void tmem_ld2_16x256b_x4_wait(uint32_t a0, uint32_t a1, uint32_t (&r)[2][16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[0][4]), "=r"(r[0][5]), "=r"(r[0][6]),
        "=r"(r[0][7]), "=r"(r[0][8]), "=r"(r[0][9]), "=r"(r[0][10]), "=r"(r[0][11]), "=r"(r[0][12]),
        "=r"(r[0][13]), "=r"(r[0][14]), "=r"(r[0][15]),
        "=r"(r[1][0]), "=r"(r[1][1]), "=r"(r[1][2]), "=r"(r[1][3]), "=r"(r[1][4]), "=r"(r[1][5]), "=r"(r[1][6]),
        "=r"(r[1][7]), "=r"(r[1][8]), "=r"(r[1][9]), "=r"(r[1][10]), "=r"(r[1][11]), "=r"(r[1][12]),
        "=r"(r[1][13]), "=r"(r[1][14]), "=r"(r[1][15])
      : "r"(a0), "r"(a1)
      : "memory");
}

}  // namespace dsa
