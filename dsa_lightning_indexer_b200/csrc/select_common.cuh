// Block-wide scans and the exact whole-row top-k select, shared by the
// selection kernels (topk_select.cu) and the fused decode tail
// (decode_tail.cu).  The select keeps the n largest (score, -position) of a
// row: score descending, ties to the lower position (llama.cpp b12180 news:
// aiaulis.com paragraphs 2-3, only the highest-scored tokens are attended).
#pragma once

#include "dsa_common.cuh"

namespace dsa {
namespace sel {

// Exclusive prefix sum over a block of NW warps, in thread order.
template <int NW>
__device__ __forceinline__ int block_excl_sum_nw(int v, int* buf /*[NW + 1]*/, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) buf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int wv = lane < NW ? buf[lane] : 0;
    int wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < NW) buf[lane] = wi - wv;
    if (lane == NW - 1) buf[NW] = wi;
  }
  __syncthreads();
  const int res = buf[warp] + incl - v;
  total = buf[NW];
  __syncthreads();
  return res;
}


// Exclusive count of `flag` over a block of NW warps, in thread order.
template <int NW>
__device__ __forceinline__ int block_excl_count_nw(bool flag, int* buf /*[NW + 1]*/, int& total) {
  const int lane = threadIdx.x & 31;
  const unsigned m = __ballot_sync(0xffffffffu, flag);
  const int res = block_excl_sum_nw<NW>(lane == 0 ? __popc(m) : 0, buf, total);
  // res counts whole warps before this one (lane 0 carried each warp's count)
  const int before_warp = __shfl_sync(0xffffffffu, res, 0);
  return before_warp + __popc(m & ((1u << lane) - 1u));
}

// Exact top-k of one row read from global memory, by a block of NW warps:
// three MSB radix passes (11 + 11 + 10 bits) re-reading the row, then an
// ordered emission of keys > theta and the first ties at theta.
template <int NW>
__device__ void row_select_global(const float* sc, int n, int k, int32_t* out, int* hist,
                                  int* buf) {
  constexpr int NT = NW * 32;
  __shared__ int pick_digit_g, pick_above_g;
  uint32_t prefix = 0, pmask = 0;
  int remaining = k;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass == 2 ? 0x3FFu : 0x7FFu;
    for (int i = threadIdx.x; i < 2048; i += NT) hist[i] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < n; s += NT) {
      const uint32_t key = score_key(sc[s]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1);
    }
    __syncthreads();
    // Thread t looks at the digits of group u = NT-1-t (2048/NT digits each),
    // so the exclusive prefix in thread order counts keys in higher digits.
    constexpr int D = 2048 / NT;
    const int u = NT - 1 - static_cast<int>(threadIdx.x);
    int cnt[D];
    int tot = 0;
#pragma unroll
    for (int j = 0; j < D; ++j) {
      cnt[j] = hist[D * u + j];
      tot += cnt[j];
    }
    int total;
    int above = block_excl_sum_nw<NW>(tot, buf, total);
    if (above < remaining && remaining <= above + tot) {
#pragma unroll
      for (int j = D - 1; j >= 0; --j) {
        if (above + cnt[j] >= remaining) {
          pick_digit_g = D * u + j;
          pick_above_g = above;
          break;
        }
        above += cnt[j];
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(pick_digit_g) << shift;
    pmask |= dmask << shift;
    remaining -= pick_above_g;
    __syncthreads();
  }
  const uint32_t theta = prefix;
  const int need = remaining;
  int taken_eq = 0, out_pos = 0;
#pragma unroll 1
  for (int base = 0; base < n && out_pos < k; base += NT) {
    const int s = base + static_cast<int>(threadIdx.x);
    const bool valid = s < n;
    const uint32_t key = valid ? score_key(sc[s]) : 0u;
    const bool gt = valid && key > theta;
    const bool eq = valid && key == theta;
    int eq_total, sel_total;
    const int eq_rank = taken_eq + block_excl_count_nw<NW>(eq, buf, eq_total);
    const bool sel = gt || (eq && eq_rank < need);
    const int slot = out_pos + block_excl_count_nw<NW>(sel, buf, sel_total);
    if (sel) out[slot] = s;
    taken_eq += eq_total;
    out_pos += sel_total;
  }
}

}  // namespace sel
}  // namespace dsa
