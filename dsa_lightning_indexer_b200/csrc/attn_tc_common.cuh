// Pieces shared by the two tcgen05 attention kernels (many-row tiles and
// single-tile decode slices): launch parameters, shared-memory descriptors
// and TMEM access, fast exp2, named barriers, and the per-row sequence
// lookup.
#pragma once

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace attn_tc {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct TcParams {
  const int32_t* q_offsets;
  CacheLayout cache;
  const int32_t* ctx_lens;
  const __nv_bfloat16* kv;
  const int32_t* idx;
  float* out;
  float* lse;
  unsigned* err;
  float* part_o;        // [n_split][Nq][H][512] unnormalised slice outputs (n_split > 1)
  float2* part_ml;      // [n_split][Nq][H] (running max in log2 units, row sum)
  int B, Nq, H, top_k;
  int n_split, split_len;  // slices of the selected set, slots per slice
  int idx_prefix;       // valid entries are the first min(top_k, p+1) slots
  int batch_ready;      // the batch arrays may be read before the dependent-launch wait
  float scale_log2;
  const __nv_bfloat16* q;  // [Nq][H][576] queries (the kernels that read them directly)
  int wave;                // CTAs resident at once (one per SM): the many-row kernel
                           // prefetches for row r + wave
};

// MN-major operand in the 128-byte swizzle layout: 64-element chunks along
// M/N `lbo` bytes apart, groups of 8 K-rows 1024 bytes apart.
__device__ __forceinline__ uint64_t sdesc_sw128_mn(uint32_t saddr, uint32_t lbo) {
  uint64_t d = static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// 16x32bx2 shape: threads 0-15 read TMEM lanes base..base+15 at the given
// column, threads 16-31 the same lanes kSplit columns further.  With the
// M = 64 accumulator layout (head row 16q + j at lane 32q + j) the two half
// warps split each head row's logits between them.
template <int kSplit>
__device__ __forceinline__ void tmem_ld_16x32bx2_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16], %17;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr), "n"(kSplit));
}

template <int kSplit>
__device__ __forceinline__ void tmem_ld_16x32bx2_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
      "[%32], %33;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr), "n"(kSplit));
}

template <int kSplit>
__device__ __forceinline__ void tmem_ld_16x32bx2_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8], %9;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr), "n"(kSplit));
}

// 2^x on the special-function unit (relative error about 2^-22); 2^-inf = 0.
__device__ __forceinline__ float exp2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 16x32bx2 store: threads 0-15 write TMEM lanes base..base+15 from the
// given column, threads 16-31 the same lanes kSplit columns further.
template <int kSplit>
__device__ __forceinline__ void tmem_st_16x32bx2_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], %1, "
      "{%2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17};" ::"r"(taddr),
      "n"(kSplit), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
      "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// tcgen05.mma (kind::f16, one CTA) with the A operand read from tensor
// memory, issued by one elected lane of a converged warp: d (+)= A . B.
__device__ __forceinline__ void tc_mma_bf16_ts_warp(uint32_t d_tmem, uint32_t a_tmem,
                                                    uint64_t bdesc, uint32_t idesc,
                                                    uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void cp_async16_tc(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// OR of `pred` over the `threads` threads meeting at named barrier `id`.
__device__ __forceinline__ bool named_bar_or(int id, int threads, bool pred) {
  uint32_t res;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(res)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(threads)
      : "memory");
  return res != 0;
}

// Sequence facts of query row r, looked up by each warp with all of its
// loads in flight at once (lane l checks sequences l, l + 32, ...): where the
// sequence's positions live in the caches and the row's causal length p + 1.
struct RowSeq {
  SeqRows rows;
  int len;
};

__device__ __forceinline__ RowSeq row_seq_warp(const int32_t* q_offsets, const CacheLayout& cache,
                                               const int32_t* ctx_lens, int B, int r) {
  long long kv0 = 0;
  int len = 0, hit = 0, seq = 0;
  for (int b = threadIdx.x & 31; b < B; b += 32) {
    const int q0 = __ldg(q_offsets + b), q1 = __ldg(q_offsets + b + 1);
    const long long k0 = cache.block_table ? 0 : __ldg(cache.kv_offsets + b);
    const int L = __ldg(ctx_lens + b);
    if (r >= q0 && r < q1) {
      kv0 = k0;
      len = L - (q1 - q0) + (r - q0) + 1;
      hit = 1;
      seq = b;
    }
  }
  const unsigned m = __ballot_sync(0xffffffffu, hit);
  const int src = m ? __ffs(m) - 1 : 0;
  RowSeq rs;
  rs.len = __shfl_sync(0xffffffffu, len, src);
  rs.rows = seq_rows(cache, __shfl_sync(0xffffffffu, seq, src),
                     __shfl_sync(0xffffffffu, kv0, src));
  return rs;
}

__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Starts a bulk copy of `bytes` (a multiple of 16) of shared memory at `src`
// to global `dst` (16-byte aligned).
__device__ __forceinline__ void bulk_store_issue(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile(
      "cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n\t"
      "cp.async.bulk.commit_group;" ::"l"(dst),
      "r"(src), "r"(bytes)
      : "memory");
}

// Waits until all committed bulk copies have finished reading shared memory
// (their global writes may still be in flight; they complete before the
// grid does).
__device__ __forceinline__ void bulk_wait_all_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

}  // namespace attn_tc
}  // namespace dsa
