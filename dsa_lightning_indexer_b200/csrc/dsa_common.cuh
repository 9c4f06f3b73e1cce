// Device-side building blocks shared by the DSA kernels (sm_100a only):
// mbarrier waits with a time limit, TMA tile loads, tcgen05 MMA / TMEM access,
// shared-memory matrix descriptors, and the workspace control block.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dsa {

constexpr int kIdxHeads = 32;    // indexer heads
constexpr int kIdxDim = 128;     // indexer head dim
constexpr int kLatent = 576;     // latent key row (K)
constexpr int kValue = 512;      // value width (leading part of the latent row)
constexpr int kMaxTopK = 2048;
constexpr int kMaxHeads = 128;
constexpr int kMaxSeqPerLaunch = 64;
// Score-key histogram fused into the indexer for the top-k filter: the top
// 12 bits of the order-preserving key.
constexpr int kHistShift = 20;
constexpr int kHistBins = 1 << (32 - kHistShift);

// Error bits in the workspace control block.
constexpr unsigned kErrTimeout = 1u;  // a bounded wait ran out
constexpr unsigned kErrIndex = 2u;    // an index entry outside [-1, p] was dropped

// First 256 bytes of every workspace.
struct Control {
  unsigned int err;        // OR of kErr* bits set by kernels
  unsigned int pad[63];
};
constexpr size_t kControlBytes = sizeof(Control);
static_assert(kControlBytes == 256, "control block is 256 bytes");

// About one second at B200 clocks: long enough never to fire on a healthy
// pipeline, short enough that a broken one returns control to the host.
constexpr long long kWaitCycles = 2000000000LL;

// Where the positions of a batch's sequences live in the caches: contiguous
// rows from kv_offsets[b], or pages of 2^page_shift rows listed in
// block_table[b * max_blocks ...] (block_table non-null).
struct CacheLayout {
  const int64_t* kv_offsets;   // device (contiguous caches)
  const int32_t* block_table;  // device (paged caches) or null
  int max_blocks;
  int page_shift;
};

// One sequence's part of a CacheLayout.
struct SeqRows {
  long long kv0;       // contiguous: the sequence's first row
  const int32_t* bt;   // paged: its block-table row, else null
  int page_shift;
};

__device__ __forceinline__ SeqRows seq_rows(const CacheLayout& c, int b, long long kv0) {
  SeqRows s;
  s.page_shift = c.page_shift;
  s.bt = c.block_table ? c.block_table + static_cast<size_t>(b) * c.max_blocks : nullptr;
  s.kv0 = c.block_table ? 0 : kv0;
  return s;
}

// Cache row of position `pos` of the sequence.
__device__ __forceinline__ long long seq_row(const SeqRows& s, int pos) {
  if (s.bt == nullptr) return s.kv0 + pos;
  return (static_cast<long long>(__ldg(s.bt + (pos >> s.page_shift))) << s.page_shift) |
         static_cast<long long>(pos & ((1 << s.page_shift) - 1));
}

// (a, b) = (wa, wb) * (xa, xb) + (a, b) as one paired fp32 FMA; each lane is
// an fma rounded to nearest, the same result as fmaf.
__device__ __forceinline__ void ffma2(float& a, float& b, float wa, float wb, float xa, float xb) {
  asm("{\n\t.reg .b64 acc, w, x;\n\t"
      "mov.b64 acc, {%0, %1};\n\t"
      "mov.b64 w, {%2, %3};\n\t"
      "mov.b64 x, {%4, %5};\n\t"
      "fma.rn.f32x2 acc, w, x, acc;\n\t"
      "mov.b64 {%0, %1}, acc;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(wa), "f"(wb), "f"(xa), "f"(xb));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------ mbarrier ----

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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

// Non-blocking: true if the phase of parity `parity` has completed, without
// the potential suspension of try_wait (for loops that poll several
// barriers and must not sleep on one of them).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase of parity `parity` to complete.  Gives up after
// kWaitCycles (or as soon as another thread has recorded an error), sets the
// timeout bit and returns false; the caller then abandons its loop.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (unsigned it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*reinterpret_cast<volatile unsigned*>(err) != 0u) return false;
      if (clock64() - t0 > kWaitCycles) {
        atomicOr(err, kErrTimeout);
        return false;
      }
    }
  }
}

// Waits, with the same time limit but whatever the error word says, for the
// phase of parity `parity` of `bar` to complete.  A CTA that abandoned its
// loops calls this before it exits, so that no TMA copy or tcgen05 operation
// it issued is still writing its shared memory or TMEM when they are handed
// to the next CTA.  Returns false (and sets the timeout bit) if the limit
// ran out.
__device__ __forceinline__ bool mbar_drain(uint32_t bar, uint32_t parity, unsigned* err) {
  const long long t0 = clock64();
  for (unsigned it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u && clock64() - t0 > kWaitCycles) {
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
}

// True when an earlier kernel recorded an error in the workspace: the
// kernels of a call then skip their work until dsa_check_device_status
// clears the word.  Read after the dependent-launch wait.
__device__ __forceinline__ bool error_recorded(const unsigned* err) {
  return err != nullptr && *reinterpret_cast<const volatile unsigned*>(err) != 0u;
}

// ----------------------------------------------------------------- TMA ----

__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Brings a 2-D tile of the tensor into L2 (nothing is written to shared
// memory and nothing waits for it).  c0 is the innermost coordinate.
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1)
               : "memory");
}

// 2-D tiled bulk tensor load into this CTA's shared memory; completion is
// counted in bytes on `bar`.  c0 is the innermost (contiguous) coordinate.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
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

// -------------------------------------------------------------- tcgen05 ----

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
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

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulator.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same, issued from a converged warp: elect.sync picks the issuing lane
// (the lowest active one), so the warp's descriptor arithmetic stays uniform.
// Much cheaper per MMA than issuing from a lane-0 branch.
__device__ __forceinline__ void tc_mma_bf16_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// tc_commit from a converged warp, by the lane that tc_mma_bf16_warp elects.
__device__ __forceinline__ void tc_commit_warp(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          bar)
      : "memory");
}

// Instruction descriptor, kind::f16: bf16 A and B (both K-major), fp32 D.
// Bits: [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B
// format (1 = bf16), [15] A major, [16] B major (0 = K), [17,23) N >> 3,
// [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a K-major operand stored in the
// 128-byte swizzle layout that TMA writes for a box whose rows are 128 bytes:
// rows of 128 B, groups of 8 rows 1024 B apart (stride byte offset), the
// leading byte offset unused.  Bits: [0,14) address >> 4, [16,30) LBO >> 4,
// [32,46) SBO >> 4, [46,48) version 1, [61,64) layout 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------- dependent launches ----

// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialization attribute may start while its predecessor finishes;
// it must call pdl_wait() before touching memory the predecessor writes or
// reads.  Both are no-ops for an ordinary launch.
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------- helpers ----

// Order-preserving map of an fp32 score to uint32 (larger score, larger key);
// -0 is mapped like +0.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

__device__ __forceinline__ int warp_id_uniform() {
  return __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) / 32, 0);
}

}  // namespace dsa
