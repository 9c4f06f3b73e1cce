// Attention over the selected rows of the shared latent cache.
//
//   O[q, g, :] = sum_{s in S_q} softmax_s( scale * q[q, g, :] . kv[s, :] ) * kv[s, :512]
//
// (llama.cpp b12180 news: aiaulis.com paragraph 2 — attention is computed only
// for the selected tokens; devotd.net section 2 — a key-only cache per DSA
// layer, whose leading 512 entries serve as V.)
//
// Only the selected rows are read: each row is gathered once per CTA with
// 16-byte cp.async copies into shared memory (double-buffered tiles of 32
// rows) and used for both Q.K^T and P.V.  A CTA owns one query row, a block of
// heads (16 per warp group of four warps) and a contiguous slice of the
// selected set.  With few rows (decode) it takes 16 heads and a slice of the
// set; a second kernel, spread over the whole GPU, merges the slices' partial
// results with the log-sum-exp rule.  (Many-row launches use the tcgen05
// kernel in sparse_attn_tc.cu.)  Softmax runs online in fp32 in base 2.  P
// enters the P.V product as bf16 hi + lo parts, so its rounding error stays
// near 2^-16 relative.
#include <algorithm>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kTileRows = 32;                  // gathered rows per tile
constexpr int kRowPad = kLatent + 8;           // 584 bf16 = 1168 B per smem row
constexpr int kPPad = kTileRows + 8;           // P row stride (bf16)
constexpr int kHeadsPerCta = 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct AttnParams {
  const int32_t* q_offsets;
  CacheLayout cache;
  const int32_t* ctx_lens;
  unsigned* err;        // error word for dropped index entries, or null
  const __nv_bfloat16* q;
  const __nv_bfloat16* kv;
  const int32_t* idx;
  float* out;
  float* lse;
  float* part_o;        // [n_split][Nq][H][512] unnormalised slice outputs
  float2* part_ml;      // [n_split][Nq][H] (running max in log2 units, row sum)
  int B, Nq, H, top_k, n_split, split_len;
  float scale_log2;     // scale * log2(e)
};

__device__ __forceinline__ int owner_seq(const int32_t* q_offsets, int B, int r) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (q_offsets[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A(16x16, row) * B(16x8, col), bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void named_bar(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <int NG>  // warp groups of 16 heads (4 warps each)
__global__ void __launch_bounds__(NG * 128, 1) sparse_attn_kernel(const AttnParams P) {
  constexpr int HB = NG * 16;
  constexpr int kThreads = NG * 128;
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16* const Qs = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* const KVs = Qs + HB * kRowPad;                    // [2][kTileRows][kRowPad]
  __nv_bfloat16* const Ph = KVs + 2 * kTileRows * kRowPad;          // [HB][kPPad]
  __nv_bfloat16* const Pl = Ph + HB * kPPad;
  float* const red = reinterpret_cast<float*>(Pl + HB * kPPad);     // [HB][4]
  int* const tidx = reinterpret_cast<int*>(red + HB * 4);          // [2][kTileRows]

  const int r = blockIdx.x;
  const int h0 = blockIdx.y * HB;
  const int sp = blockIdx.z;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int hg = warp >> 2, qd = warp & 3;
  const int g = lane >> 2, c = lane & 3;

  pdl_wait();
  pdl_launch_dependents();
  const int b = owner_seq(P.q_offsets, P.B, r);
  const SeqRows sr = seq_rows(P.cache, b, P.cache.block_table ? 0 : P.cache.kv_offsets[b]);
  // Causal length p + 1 of the row: only positions below it are read.
  const int row_len = P.ctx_lens[b] - (P.q_offsets[b + 1] - P.q_offsets[b]) +
                      (r - P.q_offsets[b]) + 1;
  const int32_t* const idx_row = P.idx + static_cast<size_t>(r) * P.top_k;
  const int slot0 = sp * P.split_len;
  const int slot1 = min(slot0 + P.split_len, P.top_k);
  const int n_tiles = slot1 > slot0 ? (slot1 - slot0 + kTileRows - 1) / kTileRows : 0;

  // Q rows of this head block -> smem (zero rows past H).
  for (int e = tid; e < HB * (kLatent / 8); e += kThreads) {
    const int h = e / (kLatent / 8), ch = e - h * (kLatent / 8);
    const uint32_t dst = smem_u32(Qs + h * kRowPad + ch * 8);
    if (h0 + h < P.H) {
      cp_async16(dst, P.q + (static_cast<size_t>(r) * P.H + h0 + h) * kLatent + ch * 8);
    } else {
      *reinterpret_cast<uint4*>(Qs + h * kRowPad + ch * 8) = make_uint4(0, 0, 0, 0);
    }
  }

  auto load_tile = [&](int t, int buf) {
    const int s0 = slot0 + t * kTileRows;
    __nv_bfloat16* const dstb = KVs + buf * kTileRows * kRowPad;
    for (int e = tid; e < kTileRows * (kLatent / 8); e += kThreads) {
      const int i = e / (kLatent / 8), ch = e - i * (kLatent / 8);
      const int slot = s0 + i;
      int pos = slot < slot1 ? __ldg(idx_row + slot) : -1;
      if (pos < -1 || pos >= row_len) {  // outside 0..p: skipped (and recorded)
        if (P.err != nullptr && ch == 0) atomicOr(P.err, kErrIndex);
        pos = -1;
      }
      if (ch == 0) tidx[buf * kTileRows + i] = pos;
      if (pos >= 0) {
        cp_async16(smem_u32(dstb + i * kRowPad + ch * 8),
                   P.kv + static_cast<size_t>(seq_row(sr, pos)) * kLatent + ch * 8);
      } else {
        *reinterpret_cast<uint4*>(dstb + i * kRowPad + ch * 8) = make_uint4(0, 0, 0, 0);
      }
    }
  };

  if (n_tiles > 0) load_tile(0, 0);
  cp_async_commit();

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_g = -INFINITY, m_g8 = -INFINITY;   // running max (log2 units), rows g and g+8
  float l_g = 0.f, l_g8 = 0.f;               // this thread's share of the row sums

  const int hrow = hg * 16;  // first head row of this warp group in smem
  const uint32_t q_base = smem_u32(Qs);
  const uint32_t ph_base = smem_u32(Ph), pl_base = smem_u32(Pl);

  for (int t = 0; t < n_tiles; ++t) {
    const int buf = t & 1;
    if (t + 1 < n_tiles) load_tile(t + 1, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    const __nv_bfloat16* const kvb = KVs + buf * kTileRows * kRowPad;
    const uint32_t kv_base = smem_u32(kvb);
    // ---- S = Q K^T for heads hrow..+15 and tile rows qd*8..+7 ------------
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    float s_odd[4] = {0.f, 0.f, 0.f, 0.f};  // second chain halves the MMA dependency depth
    {
      const uint32_t a_addr = q_base + ((hrow + (lane & 15)) * kRowPad + (lane >> 4) * 8) * 2;
      const uint32_t b_addr = kv_base + ((qd * 8 + (lane & 7)) * kRowPad + (lane >> 3) * 8) * 2;
#pragma unroll 6
      for (int ks = 0; ks < kLatent / 32; ++ks) {
        uint32_t a0, a1, a2, a3, a4, a5, a6, a7, b0, b1, b2, b3;
        ldsm_x4(a_addr + ks * 64, a0, a1, a2, a3);
        ldsm_x4(a_addr + ks * 64 + 32, a4, a5, a6, a7);
        ldsm_x4(b_addr + ks * 64, b0, b1, b2, b3);
        mma_bf16_16816(s, a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(s_odd, a4, a5, a6, a7, b2, b3);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) s[i] += s_odd[i];
    }
    const int* const ti = tidx + buf * kTileRows;
    const bool v0 = ti[qd * 8 + 2 * c] >= 0, v1 = ti[qd * 8 + 2 * c + 1] >= 0;
    s[0] = v0 ? s[0] * P.scale_log2 : -INFINITY;
    s[1] = v1 ? s[1] * P.scale_log2 : -INFINITY;
    s[2] = v0 ? s[2] * P.scale_log2 : -INFINITY;
    s[3] = v1 ? s[3] * P.scale_log2 : -INFINITY;
    float mx_g = fmaxf(s[0], s[1]), mx_g8 = fmaxf(s[2], s[3]);
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
      mx_g = fmaxf(mx_g, __shfl_xor_sync(0xffffffffu, mx_g, o2));
      mx_g8 = fmaxf(mx_g8, __shfl_xor_sync(0xffffffffu, mx_g8, o2));
    }
    if (c == 0) {
      red[(hrow + g) * 4 + qd] = mx_g;
      red[(hrow + g + 8) * 4 + qd] = mx_g8;
    }
    named_bar(1 + hg, 128);
    const float tm_g = fmaxf(fmaxf(red[(hrow + g) * 4 + 0], red[(hrow + g) * 4 + 1]),
                             fmaxf(red[(hrow + g) * 4 + 2], red[(hrow + g) * 4 + 3]));
    const float tm_g8 = fmaxf(fmaxf(red[(hrow + g + 8) * 4 + 0], red[(hrow + g + 8) * 4 + 1]),
                              fmaxf(red[(hrow + g + 8) * 4 + 2], red[(hrow + g + 8) * 4 + 3]));
    const float mn_g = fmaxf(m_g, tm_g), mn_g8 = fmaxf(m_g8, tm_g8);
    const float al_g = mn_g == -INFINITY ? 1.f : exp2f(m_g - mn_g);
    const float al_g8 = mn_g8 == -INFINITY ? 1.f : exp2f(m_g8 - mn_g8);
    m_g = mn_g;
    m_g8 = mn_g8;
    const float p0 = s[0] == -INFINITY ? 0.f : exp2f(s[0] - mn_g);
    const float p1 = s[1] == -INFINITY ? 0.f : exp2f(s[1] - mn_g);
    const float p2 = s[2] == -INFINITY ? 0.f : exp2f(s[2] - mn_g8);
    const float p3 = s[3] == -INFINITY ? 0.f : exp2f(s[3] - mn_g8);
    l_g = l_g * al_g + (p0 + p1);
    l_g8 = l_g8 * al_g8 + (p2 + p3);
    {
      const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
      const __nv_bfloat162 hb01 = *reinterpret_cast<const __nv_bfloat162*>(&h01);
      const __nv_bfloat162 hb23 = *reinterpret_cast<const __nv_bfloat162*>(&h23);
      const uint32_t l01 = pack_bf16x2(p0 - __low2float(hb01), p1 - __high2float(hb01));
      const uint32_t l23 = pack_bf16x2(p2 - __low2float(hb23), p3 - __high2float(hb23));
      const int col = qd * 8 + 2 * c;
      *reinterpret_cast<uint32_t*>(Ph + (hrow + g) * kPPad + col) = h01;
      *reinterpret_cast<uint32_t*>(Ph + (hrow + g + 8) * kPPad + col) = h23;
      *reinterpret_cast<uint32_t*>(Pl + (hrow + g) * kPPad + col) = l01;
      *reinterpret_cast<uint32_t*>(Pl + (hrow + g + 8) * kPPad + col) = l23;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= al_g;
      o[i][1] *= al_g;
      o[i][2] *= al_g8;
      o[i][3] *= al_g8;
    }
    named_bar(1 + hg, 128);

    // ---- O[heads, dv qd*128..+127] += P V ------------------------------
#pragma unroll
    for (int kk = 0; kk < kTileRows / 16; ++kk) {
      uint32_t ah0, ah1, ah2, ah3, al0, al1, al2, al3;
      const uint32_t pa = ((hrow + (lane & 15)) * kPPad + kk * 16 + (lane >> 4) * 8) * 2;
      ldsm_x4(ph_base + pa, ah0, ah1, ah2, ah3);
      ldsm_x4(pl_base + pa, al0, al1, al2, al3);
      const uint32_t vrow = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(kv_base + (vrow * kRowPad + qd * 128 + np * 16 + (lane >> 4) * 8) * 2, b0, b1,
                  b2, b3);
        mma_bf16_16816(o[2 * np], ah0, ah1, ah2, ah3, b0, b1);
        mma_bf16_16816(o[2 * np], al0, al1, al2, al3, b0, b1);
        mma_bf16_16816(o[2 * np + 1], ah0, ah1, ah2, ah3, b2, b3);
        mma_bf16_16816(o[2 * np + 1], al0, al1, al2, al3, b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // ---- row sums across the quad and the four warps of the group --------
#pragma unroll
  for (int o2 = 1; o2 < 4; o2 <<= 1) {
    l_g += __shfl_xor_sync(0xffffffffu, l_g, o2);
    l_g8 += __shfl_xor_sync(0xffffffffu, l_g8, o2);
  }
  __syncthreads();
  if (c == 0) {
    red[(hrow + g) * 4 + qd] = l_g;
    red[(hrow + g + 8) * 4 + qd] = l_g8;
  }
  __syncthreads();
  const float L_g = (red[(hrow + g) * 4 + 0] + red[(hrow + g) * 4 + 1]) +
                    (red[(hrow + g) * 4 + 2] + red[(hrow + g) * 4 + 3]);
  const float L_g8 = (red[(hrow + g + 8) * 4 + 0] + red[(hrow + g + 8) * 4 + 1]) +
                     (red[(hrow + g + 8) * 4 + 2] + red[(hrow + g + 8) * 4 + 3]);

  const int ha = h0 + hrow + g, hb8 = ha + 8;
  if (P.n_split == 1) {
    const float inv_g = L_g > 0.f ? 1.f / L_g : 0.f;
    const float inv_g8 = L_g8 > 0.f ? 1.f / L_g8 : 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int dv = qd * 128 + i * 8 + 2 * c;
      if (ha < P.H)
        *reinterpret_cast<float2*>(P.out + (static_cast<size_t>(r) * P.H + ha) * kValue + dv) =
            make_float2(o[i][0] * inv_g, o[i][1] * inv_g);
      if (hb8 < P.H)
        *reinterpret_cast<float2*>(P.out + (static_cast<size_t>(r) * P.H + hb8) * kValue + dv) =
            make_float2(o[i][2] * inv_g8, o[i][3] * inv_g8);
    }
    if (P.lse && qd == 0 && c == 0) {
      if (ha < P.H)
        P.lse[static_cast<size_t>(r) * P.H + ha] = L_g > 0.f ? (m_g + log2f(L_g)) * kLn2 : -INFINITY;
      if (hb8 < P.H)
        P.lse[static_cast<size_t>(r) * P.H + hb8] =
            L_g8 > 0.f ? (m_g8 + log2f(L_g8)) * kLn2 : -INFINITY;
    }
  } else {
    const size_t rec = (static_cast<size_t>(sp) * P.Nq + r) * P.H;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int dv = qd * 128 + i * 8 + 2 * c;
      if (ha < P.H)
        *reinterpret_cast<float2*>(P.part_o + (rec + ha) * kValue + dv) =
            make_float2(o[i][0], o[i][1]);
      if (hb8 < P.H)
        *reinterpret_cast<float2*>(P.part_o + (rec + hb8) * kValue + dv) =
            make_float2(o[i][2], o[i][3]);
    }
    if (qd == 0 && c == 0) {
      if (ha < P.H) P.part_ml[rec + ha] = make_float2(m_g, L_g);
      if (hb8 < P.H) P.part_ml[rec + hb8] = make_float2(m_g8, L_g8);
    }
  }
}

// Merges the slices of one (query row, head): O = sum_s 2^(m_s - M) O_s /
// sum_s 2^(m_s - M) l_s.  One CTA per (row, head), one float4 of O per thread;
// the slices' loads are independent so they overlap.
constexpr int kMaxSplit = 64;
__global__ void __launch_bounds__(128) attn_merge_kernel(const AttnParams P) {
  __shared__ float wgt[kMaxSplit];
  __shared__ float inv_total, lse_val;
  pdl_wait();
  pdl_launch_dependents();
  const int r = blockIdx.x, h = blockIdx.y;
  const size_t rec = static_cast<size_t>(r) * P.H + h;
  const size_t stride = static_cast<size_t>(P.Nq) * P.H;
  // Every slice's part of this thread's 4 value dims is requested up front
  // (up to kBatch slices), so the loads overlap the weights' computation.
  constexpr int kBatch = 32;
  const int dv = threadIdx.x * 4;
  const float* const po = P.part_o + rec * kValue + dv;
  float4 x[kBatch];
#pragma unroll
  for (int j = 0; j < kBatch; ++j) {
    x[j] = j < P.n_split ? __ldcg(reinterpret_cast<const float4*>(po + j * stride * kValue))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (threadIdx.x < 32) {
    float m[kMaxSplit / 32], l[kMaxSplit / 32];
    float M = -INFINITY;
#pragma unroll
    for (int j = 0; j < kMaxSplit / 32; ++j) {
      const int sp = threadIdx.x + 32 * j;
      const float2 ml = sp < P.n_split ? __ldcg(P.part_ml + sp * stride + rec)
                                       : make_float2(-INFINITY, 0.f);
      m[j] = ml.x;
      l[j] = ml.y;
      M = fmaxf(M, ml.x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxSplit / 32; ++j) {
      const float w = m[j] == -INFINITY ? 0.f : exp2f(m[j] - M);
      const int sp = threadIdx.x + 32 * j;
      if (sp < P.n_split) wgt[sp] = w;
      L += w * l[j];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (threadIdx.x == 0) {
      inv_total = L > 0.f ? 1.f / L : 0.f;
      lse_val = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
  }
  __syncthreads();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < kBatch; ++j) {
    const float w = j < P.n_split ? wgt[j] : 0.f;
    acc.x = fmaf(w, x[j].x, acc.x);
    acc.y = fmaf(w, x[j].y, acc.y);
    acc.z = fmaf(w, x[j].z, acc.z);
    acc.w = fmaf(w, x[j].w, acc.w);
  }
  for (int sp = kBatch; sp < P.n_split; ++sp) {
    const float w = wgt[sp];
    const float4 y = __ldcg(reinterpret_cast<const float4*>(po + sp * stride * kValue));
    acc.x = fmaf(w, y.x, acc.x);
    acc.y = fmaf(w, y.y, acc.y);
    acc.z = fmaf(w, y.z, acc.z);
    acc.w = fmaf(w, y.w, acc.w);
  }
  const float inv = inv_total;
  *reinterpret_cast<float4*>(P.out + rec * kValue + dv) =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (P.lse && threadIdx.x == 0) P.lse[rec] = lse_val;
}

template <int NG>
size_t attn_smem_bytes() {
  constexpr int HB = NG * 16;
  return static_cast<size_t>(HB * kRowPad + 2 * kTileRows * kRowPad + 2 * HB * kPPad) * 2 +
         HB * 4 * sizeof(float) + 2 * kTileRows * sizeof(int);
}

template <int NG>
cudaError_t launch_ng(const AttnParams& P, int head_blocks, cudaStream_t stream) {
  const size_t smem = attn_smem_bytes<NG>();
  cudaError_t e = ensure_smem_limit<sparse_attn_kernel<NG>>(static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(sparse_attn_kernel<NG>, dim3(P.Nq, head_blocks, P.n_split), dim3(NG * 128),
                    smem, stream, 0, P);
}

}  // namespace

AttnPlan attn_plan(int Nq, int H, int top_k, int num_sms) {
  // tcgen05 kernel: 64 heads per CTA (one CTA per SM).  With few rows the
  // selected set is sliced so the GPU fills; slices hold whole 16-slot groups.
  AttnPlan p;
  p.decode = 0;
  p.tc = 1;
  p.hb = kHeadsPerCta;
  p.head_blocks = (H + kHeadsPerCta - 1) / kHeadsPerCta;
  p.n_split = 1;
  p.split_len = top_k;
  const long long base = static_cast<long long>(Nq) * p.head_blocks;
  // Few rows: one tile of selected slots per CTA, as long as that takes at
  // most two waves of one CTA per SM.
  const int slots = attn_decode_slots();
  const int n_dec = (top_k + slots - 1) / slots;
  if (base > 0 && base < num_sms && n_dec <= kMaxSplit && base * n_dec <= 2LL * num_sms) {
    p.decode = 1;
    p.n_split = n_dec;
    p.split_len = slots;
    return p;
  }
  if (base > 0 && base < num_sms) {
    const int want = static_cast<int>(num_sms / base);
    const int n = std::min(std::min(want, kMaxSplit), (top_k + 15) / 16);
    if (n > 1) {
      const int per = ((top_k + n - 1) / n + 15) / 16 * 16;
      p.n_split = (top_k + per - 1) / per;
      p.split_len = per;
    }
  }
  return p;
}

AttnPlan attn_plan_core(int Nq, int H, int top_k, int num_sms) {
  AttnPlan p;
  p.decode = 0;
  p.tc = 0;
  p.hb = std::min(kHeadsPerCta, (H + 15) / 16 * 16);
  p.head_blocks = (H + p.hb - 1) / p.hb;
  p.n_split = 1;
  const long long rows = Nq;
  if (rows * p.head_blocks < num_sms && rows > 0) {
    // Few rows: 16 heads per CTA (two CTAs fit an SM) and slices of the set.
    p.hb = 16;
    p.head_blocks = (H + 15) / 16;
    const long long base = rows * p.head_blocks;
    const int want = static_cast<int>(std::max<long long>(1, 2LL * num_sms / base));
    const int n = std::min(std::min(want, kMaxSplit), (top_k + kTileRows - 1) / kTileRows);
    if (n > 1) {
      const int per = ((top_k + n - 1) / n + kTileRows - 1) / kTileRows * kTileRows;
      p.n_split = (top_k + per - 1) / per;
    }
  }
  p.split_len = ((top_k + p.n_split - 1) / p.n_split + kTileRows - 1) / kTileRows * kTileRows;
  return p;
}

size_t attn_partial_bytes(int Nq, int H, const AttnPlan& p) {
  if (p.n_split <= 1) return 0;
  return static_cast<size_t>(p.n_split) * Nq * H * (kValue + 2) * sizeof(float);
}

cudaError_t launch_sparse_attn(const AttnArgs& a, cudaStream_t stream) {
  if (a.Nq == 0) return cudaSuccess;
  if (a.plan.decode) return launch_sparse_attn_decode(a, stream);
  if (a.plan.tc) return launch_sparse_attn_tc(a, stream);
  AttnParams P;
  P.q_offsets = a.q_offsets;
  P.cache = a.cache;
  P.ctx_lens = a.ctx_lens;
  P.err = a.err;
  P.q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  P.kv = reinterpret_cast<const __nv_bfloat16*>(a.kv);
  P.idx = a.idx;
  P.out = a.out;
  P.lse = a.lse;
  const size_t n_rec = static_cast<size_t>(a.plan.n_split) * a.Nq * a.H;
  P.part_o = a.part;
  P.part_ml = reinterpret_cast<float2*>(a.part + n_rec * kValue);
  P.B = a.B;
  P.Nq = a.Nq;
  P.H = a.H;
  P.top_k = a.top_k;
  P.n_split = a.plan.n_split;
  P.split_len = a.plan.split_len;
  P.scale_log2 = a.scale * kLog2e;
  cudaError_t e;
  switch (a.plan.hb / 16) {
    case 1: e = launch_ng<1>(P, a.plan.head_blocks, stream); break;
    case 2: e = launch_ng<2>(P, a.plan.head_blocks, stream); break;
    case 3: e = launch_ng<3>(P, a.plan.head_blocks, stream); break;
    default: e = launch_ng<4>(P, a.plan.head_blocks, stream); break;
  }
  if (e != cudaSuccess || P.n_split == 1) return e;
  return launch_pdl(attn_merge_kernel, dim3(a.Nq, a.H), dim3(128), 0, stream, 0, P);
}

cudaError_t launch_attn_merge(const AttnArgs& a, cudaStream_t stream) {
  AttnParams P = {};
  P.Nq = a.Nq;
  P.H = a.H;
  P.n_split = a.plan.n_split;
  const size_t n_rec = static_cast<size_t>(a.plan.n_split) * a.Nq * a.H;
  P.part_o = a.part;
  P.part_ml = reinterpret_cast<float2*>(a.part + n_rec * kValue);
  P.out = a.out;
  P.lse = a.lse;
  return launch_pdl(attn_merge_kernel, dim3(a.Nq, a.H), dim3(128), 0, stream, 0, P);
}

}  // namespace dsa
