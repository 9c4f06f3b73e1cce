// Attention over the selected latent rows for few query rows (decode), on
// tcgen05 tensor cores: one CTA per (query row, 64-head block, slice of 64
// selected slots), a single gathered tile per CTA.
//
//   S   = Q[64 heads, 576] . K_tile[64, 576]^T       M = 64,  N = 64, K = 576
//   O^T = V_tile^T[512, 64] . P^T[64, 64 heads]      M = 128 (x4), N = 64, K = 64
//
// (llama.cpp b12180 news: aiaulis.com paragraph 2 — attention only over the
// selected tokens; devotd.net section 2 — one key-only latent cache whose
// leading 512 entries serve as V.)
//
// With one tile there is no running maximum to carry: P = 2^(s - m) with the
// tile's own maximum m, and the slice's unnormalised O with (m, sum) goes to
// the merge (or, for a single slice, O / sum and the log-sum-exp go straight
// to the output).  All four gather warps copy the one tile, so its rows are
// requested as fast as the load/store unit takes them; the tile is stored in
// the 128-byte swizzled layout and read by both products (K-major for S,
// MN-major for O^T).  P is bf16 hi + lo (two MMAs).  The result rows of the
// 64 heads are contiguous, so they are staged in the freed Q / tile space and
// leave in one bulk copy.
//
// Warp roles (288 threads): warps 0-3 softmax and output (TMEM quadrants
// 0-3), warp 4 TMEM allocation, the Q load (TMA) and MMA issue (converged
// warp, one elected lane), warps 5-8 the gather.
#include "attn_tc_common.cuh"

namespace dsa {
namespace {

using namespace attn_tc;

constexpr int kTD = 64;                   // selected slots per CTA (one tile)
constexpr int kHB = 64;                   // heads per CTA
constexpr int kBoxes = kLatent / 64;
constexpr int kQBox = kHB * 128;
constexpr int kKVBox = kTD * 128;
constexpr int kPBuf = kHB * 128;          // P^T operand: 64 heads x 64 keys bf16
constexpr int kThreads = 288;
constexpr int kSoftThreads = 128;
constexpr int kGatherThreads = 128;

constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kBoxes * kQBox;
constexpr int kOffP = kOffKV + kBoxes * kKVBox;          // [hi, lo]
constexpr int kOffStage = 0;                             // [64][512] fp32 over Q and the tile
constexpr int kOffBar = kOffP + 2 * kPBuf;
constexpr int kNumBars = 6;
constexpr int kOffTmem = kOffBar + 8 * kNumBars;
constexpr int kOffIdx = kOffTmem + 16;                   // [64] int
constexpr int kOffM = kOffIdx + kTD * 4;                 // [64] float
constexpr int kOffL = kOffM + kHB * 4;                   // [64] float
constexpr int kSmemUsed = kOffL + kHB * 4;
constexpr int kSmemBytes = kSmemUsed + 1024;
static_assert(kOffStage + kHB * kValue * 4 <= kOffP, "output staging overlaps P");
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;     // S: 64 columns (M = 64 layout)
constexpr uint32_t kColO = 64;    // O^T blocks at 64, 128, 192, 256
constexpr uint32_t kIdescS = idesc_bf16_f32(64, kTD);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kHB) | (1u << 15);  // A MN-major
constexpr int kHalf = kTD / 2;    // logits per half warp

__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_decode_kernel(const __grid_constant__ CUtensorMap qmap, const TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const bp = smem_raw + (base - raw);
  const uint32_t sQ = base + kOffQ, sKV = base + kOffKV, sP = base + kOffP;
  const uint32_t bars = base + kOffBar;
  const uint32_t b_qfull = bars, b_kvfull = bars + 8u, b_sfull = bars + 16u,
                 b_pfull = bars + 24u, b_odone = bars + 32u, b_drain = bars + 40u;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(bp + kOffTmem);
  int* const tidx = reinterpret_cast<int*>(bp + kOffIdx);
  float* const rl_s = reinterpret_cast<float*>(bp + kOffL);  // 1 / row sum per head

  const int warp = warp_id_uniform();
  const int lane = lane_id();
  const int r = blockIdx.x;
  const int h0 = blockIdx.y * kHB;
  const int sp = blockIdx.z;

  if (threadIdx.x == 0) {
    mbar_init(b_qfull, 1);
    mbar_init(b_kvfull, kGatherThreads);
    mbar_init(b_sfull, 1);
    mbar_init(b_pfull, kSoftThreads);
    mbar_init(b_odone, 1);
    mbar_init(b_drain, 1);
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  // Inside the layer the batch arrays are inputs no earlier kernel writes:
  // look the row up while the previous kernel finishes.
  RowSeq rs = {};
  if (P.batch_ready) rs = row_seq_warp(P.q_offsets, P.cache, P.ctx_lens, P.B, r);
  pdl_wait();
  pdl_launch_dependents();

  const int slot_lo = sp * P.split_len;
  // The gather warps request their slot entries before the row lookup
  // returns (the entries past the row's causal length are masked below).
  int pos_raw = -1;
  if (warp >= 5) {
    const int slot = slot_lo + (threadIdx.x - 160);
    if (threadIdx.x - 160 < kTD && slot < min(P.top_k, slot_lo + P.split_len)) {
      pos_raw = __ldg(P.idx + static_cast<size_t>(r) * P.top_k + slot);
    }
  }
  if (!P.batch_ready) rs = row_seq_warp(P.q_offsets, P.cache, P.ctx_lens, P.B, r);
  const int n_slots = P.idx_prefix ? min(P.top_k, rs.len) : P.top_k;
  const bool work = slot_lo < n_slots;  // block-uniform

  if (warp >= 5) {
    // ------------------------------------------------------------ gather --
    const int g = threadIdx.x - 160;  // 0..127
    if (work) {
      if (g < kTD) {
        // Only positions 0..p of the row are read; any other entry but -1 is
        // recorded as an error and skipped.
        int pos = slot_lo + g < n_slots ? pos_raw : -1;
        if (pos < -1 || pos >= rs.len) {
          atomicOr(P.err, kErrIndex);
          pos = -1;
        }
        // The slot's cache row (-1: nothing to read).
        tidx[g] = pos >= 0 ? static_cast<int>(seq_row(rs.rows, pos)) : -1;
      }
      named_bar_sync(2, kGatherThreads);
      // Thread (sub, piece) copies 16-byte piece `piece` of every box of
      // rows sub, sub + 16, ...: a warp instruction reads four whole 128-byte
      // lines, its four swizzled rows cover every shared-memory bank four
      // times, and the swizzle (row & 7 == sub & 7) is fixed per thread.
      const uint32_t piece = static_cast<uint32_t>(g & 7);
      const int sub = g >> 3;
      const uint32_t sw = (piece ^ static_cast<uint32_t>(sub & 7)) << 4;
      for (int i = sub; i < kTD; i += kGatherThreads >> 3) {
        const int row = tidx[i];
        const uint32_t dst = sKV + i * 128 + sw;
        if (row >= 0) {
          const __nv_bfloat16* src = P.kv + static_cast<size_t>(row) * kLatent + piece * 8;
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx) cp_async16_tc(dst + bx * kKVBox, src + bx * 64);
        } else {
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx) {
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst + bx * kKVBox),
                         "r"(0u)
                         : "memory");
          }
        }
      }
      asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
      fence_proxy_async_smem();
      mbar_arrive(b_kvfull);
    }
  } else if (warp == 4) {
    // ------------------------------------------------ Q load + MMA issue --
    if (lane == 0) {
      tma_prefetch_map(&qmap);
      mbar_arrive_expect_tx(b_qfull, kBoxes * kQBox);
      const uint64_t pol = l2_policy_evict_first();
      for (int j = 0; j < kBoxes; ++j) {
        tma_load_2d(sQ + j * kQBox, &qmap, b_qfull, 64 * j, r * P.H + h0, pol);
      }
    }
    __syncwarp();
    auto wait_all = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, P.err));
    };
    bool ok = wait_all(b_qfull, 0);
    if (work && ok && wait_all(b_kvfull, 0)) {
      tc_fence_after();
      const uint64_t dq = sdesc_sw128(sQ), dk = sdesc_sw128(sKV);
#pragma unroll
      for (int ks = 0; ks < kLatent / 16; ++ks) {
        const uint32_t off = (ks & 3) * 32;
        tc_mma_bf16_warp(tmem + kColS, dq + static_cast<uint64_t>(((ks >> 2) * kQBox + off) >> 4),
                         dk + static_cast<uint64_t>(((ks >> 2) * kKVBox + off) >> 4), kIdescS,
                         ks > 0 ? 1u : 0u);
      }
      tc_commit_warp(b_sfull);
      if (wait_all(b_pfull, 0)) {
        tc_fence_after();
        const uint64_t dv = sdesc_sw128_mn(sKV, kKVBox);
        const uint64_t dhi = sdesc_sw128(sP), dlo = dhi + static_cast<uint64_t>(kPBuf >> 4);
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
#pragma unroll
          for (int kk = 0; kk < kTD / 16; ++kk) {
            const uint64_t a = dv + static_cast<uint64_t>(((2 * blk) * kKVBox + kk * 2048) >> 4);
            const uint32_t d = tmem + kColO + 64u * blk;
            const uint64_t ko = static_cast<uint64_t>((kk * 32) >> 4);
            tc_mma_bf16_warp(d, a, dhi + ko, kIdescPV, kk > 0 ? 1u : 0u);
            tc_mma_bf16_warp(d, a, dlo + ko, kIdescPV, 1u);
          }
        }
        tc_commit_warp(b_odone);
      }
    }
    // Nothing this warp issued (the Q load, the MMAs) may still be running
    // when the CTA exits; immediate unless a wait above was abandoned.
    tc_commit_warp(b_drain);
    if (lane == 0) {
      mbar_drain(b_drain, 0, P.err);
      mbar_drain(b_qfull, 0, P.err);
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- softmax --
    const int q = warp;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const bool owner = lane < 16;
    const int hl = 16 * q + (lane & 15);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    if (work) {
      // The slot list was written by the gather warps before kv_full.
      ok = mbar_wait(b_kvfull, 0, P.err) && mbar_wait(b_sfull, 0, P.err);
      if (ok) {
        tc_fence_after();
        // This thread's half of its head row: keys k0 .. k0 + 31 of the tile.
        uint32_t va[16], vb[16];
        tmem_ld_16x32bx2_x16<kHalf>(tmem + lane_base + kColS, va);
        tmem_ld_16x32bx2_x16<kHalf>(tmem + lane_base + kColS + 16u, vb);
        tmem_ld_wait();
        const unsigned v_lo = __ballot_sync(0xffffffffu, tidx[lane] >= 0);
        const unsigned v_hi = __ballot_sync(0xffffffffu, tidx[32 + lane] >= 0);
        const int k0 = (lane >> 4) * kHalf;
        const unsigned valid = k0 == 0 ? v_lo : v_hi;
        float s[kHalf];
        float tmax = -INFINITY;
#pragma unroll
        for (int k = 0; k < kHalf; ++k) {
          const float raw_s = __uint_as_float(k < 16 ? va[k] : vb[k - 16]);
          s[k] = ((valid >> k) & 1u) ? raw_s * P.scale_log2 : -INFINITY;
          tmax = fmaxf(tmax, s[k]);
        }
        m = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
        const float m_ref = m == -INFINITY ? 0.f : m;  // masked logits give 2^-inf = 0
        float sum = 0.f;
        uint32_t hi[kHalf / 2], lo[kHalf / 2];
#pragma unroll
        for (int k = 0; k < kHalf; k += 2) {
          const float p0 = exp2_fast(s[k] - m_ref);
          const float p1 = exp2_fast(s[k + 1] - m_ref);
          sum += p0 + p1;
          const uint32_t h2 = pack2_bf16(p0, p1);
          hi[k / 2] = h2;
          lo[k / 2] = pack2_bf16(p0 - __uint_as_float(h2 << 16),
                                 p1 - __uint_as_float(h2 & 0xFFFF0000u));
        }
        l = sum + __shfl_xor_sync(0xffffffffu, sum, 16);
        const uint32_t prow_hi = sP + hl * 128;
        const uint32_t prow_lo = prow_hi + kPBuf;
#pragma unroll
        for (int j = 0; j < kHalf / 8; ++j) {
          const int c = k0 / 8 + j;
          const uint32_t off = static_cast<uint32_t>((c ^ (hl & 7)) << 4);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(prow_hi + off),
                       "r"(hi[4 * j]), "r"(hi[4 * j + 1]), "r"(hi[4 * j + 2]), "r"(hi[4 * j + 3])
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(prow_lo + off),
                       "r"(lo[4 * j]), "r"(lo[4 * j + 1]), "r"(lo[4 * j + 2]), "r"(lo[4 * j + 3])
                       : "memory");
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(b_pfull);
      }
    }
    if (owner) {
      rl_s[hl] = l > 0.f ? 1.f / l : 0.f;
    }
    // ------------------------------------------------------------ output --
    // Q and the tile are free once the products have completed (or, with no
    // work, once Q has landed): stage the 64 heads' rows there.
    if (ok) ok = work ? mbar_wait(b_odone, 0, P.err) : mbar_wait(b_qfull, 0, P.err);
    tc_fence_after();
    const bool good = !named_bar_or(1, kSoftThreads, !ok);
    if (good) {
      const bool split = P.n_split > 1;
      float* const stg = reinterpret_cast<float*>(bp + kOffStage);
      const int nh = min(kHB, P.H - h0);
      const size_t rec = split ? (static_cast<size_t>(sp) * P.Nq + r) * P.H
                               : static_cast<size_t>(r) * P.H;
      float* const dst = (split ? P.part_o : P.out) + (rec + h0) * kValue;
      // Heads 0-31, then 32-63: each half leaves in its own bulk copy while
      // the next half is staged.
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
          const int dv = 128 * blk + 32 * q + lane;
          uint32_t o[32];
          if (work) {
            tmem_ld_32x32b_x32(tmem + lane_base + kColO + 64u * blk + 32u * half, o);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int hh = 32 * half + j;
            float v = __uint_as_float(o[j]);
            if (!split) v *= rl_s[hh];
            stg[hh * kValue + dv] = v;
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, kSoftThreads);
        const int n_half = min(32, nh - 32 * half);
        if (threadIdx.x == 0 && n_half > 0) {
          bulk_store_issue(dst + static_cast<size_t>(32 * half) * kValue,
                           smem_u32(stg + 32 * half * kValue),
                           static_cast<uint32_t>(n_half * kValue * 4));
        }
      }
      if (threadIdx.x == 0) bulk_wait_all_read();
      if (owner && h0 + hl < P.H) {
        if (split) {
          P.part_ml[rec + h0 + hl] = make_float2(m, l);
        } else if (P.lse) {
          P.lse[rec + h0 + hl] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int attn_decode_slots() { return kTD; }

cudaError_t launch_sparse_attn_decode(const AttnArgs& a, cudaStream_t stream) {
  if (a.Nq == 0) return cudaSuccess;
  EncodeTiledFn fn = get_encode_tiled();
  if (!fn) return cudaErrorInvalidValue;
  CUtensorMap qmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kLatent),
                              static_cast<cuuint64_t>(a.Nq) * a.H};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kLatent) * 2};
  const cuuint32_t box[2] = {64, kHB};
  const cuuint32_t estr[2] = {1, 1};
  if (fn(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.q), dims, strides,
         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
    return cudaErrorInvalidValue;
  }
  cudaError_t e = ensure_smem_limit<sparse_attn_decode_kernel>(kSmemBytes);
  if (e != cudaSuccess) return e;
  TcParams P;
  P.q_offsets = a.q_offsets;
  P.cache = a.cache;
  P.ctx_lens = a.ctx_lens;
  P.kv = reinterpret_cast<const __nv_bfloat16*>(a.kv);
  P.idx = a.idx;
  P.out = a.out;
  P.lse = a.lse;
  P.err = a.err;
  P.idx_prefix = a.idx_prefix ? 1 : 0;
  P.batch_ready = a.batch_ready ? 1 : 0;
  P.n_split = a.plan.n_split;
  P.split_len = a.plan.split_len;
  const size_t n_rec = static_cast<size_t>(a.plan.n_split) * a.Nq * a.H;
  P.part_o = a.part;
  P.part_ml = a.part ? reinterpret_cast<float2*>(a.part + n_rec * kValue) : nullptr;
  P.B = a.B;
  P.Nq = a.Nq;
  P.H = a.H;
  P.top_k = a.top_k;
  P.scale_log2 = a.scale * kLog2e;
  P.q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  P.wave = 0;
  const int head_blocks = (a.H + kHB - 1) / kHB;
  e = launch_pdl(sparse_attn_decode_kernel, dim3(a.Nq, head_blocks, a.plan.n_split),
                 dim3(kThreads), static_cast<size_t>(kSmemBytes), stream, 0, qmap, P);
  if (e != cudaSuccess || a.plan.n_split == 1) return e;
  return launch_attn_merge(a, stream);
}

}  // namespace dsa
