// Top-k token selection per query row.
//
// Keeps the n = min(top_k, p+1) positions of 0..p with the largest
// (score, -position): score descending, ties to the lower position
// (llama.cpp b12180 news: aiaulis.com paragraphs 2-3 — only the
// highest-scored tokens are attended, 2048 of them; devotd.net configuration
// table).  Output is in ascending position order, padded with -1.
//
// Method: scores are mapped to order-preserving uint32 keys; a three-pass MSB
// radix select (11 + 11 + 10 bits, shared-memory histograms) finds the exact
// k-th largest key theta and how many of the keys equal to theta are needed;
// a final ordered pass emits every key > theta plus the first `need` keys ==
// theta, compacting with block-wide ballot prefix counts so the output is
// deterministic and sorted by position.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

struct TopkParams {
  const int32_t* q_offsets;
  const int32_t* ctx_lens;
  const float* scores;
  long long ld;
  int32_t* idx;
  int B;
  int top_k;
};

// Largest b in [0, B) with q_offsets[b] <= r: the sequence that owns row r.
__device__ __forceinline__ int owner_seq(const int32_t* q_offsets, int B, int r) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (q_offsets[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Exclusive prefix sum over the block in thread order; also returns the total.
__device__ __forceinline__ int block_excl_sum(int v, int* buf /*[kWarps + 1]*/, int& total) {
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
    const int wv = buf[lane];
    int wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    buf[lane] = wi - wv;
    if (lane == 31) buf[kWarps] = wi;
  }
  __syncthreads();
  const int res = buf[warp] + incl - v;
  total = buf[kWarps];
  __syncthreads();
  return res;
}

__device__ __forceinline__ int block_excl_count(bool flag, int* buf, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned m = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) buf[warp] = __popc(m);
  __syncthreads();
  if (warp == 0) {
    const int wv = buf[lane];
    int wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    buf[lane] = wi - wv;
    if (lane == 31) buf[kWarps] = wi;
  }
  __syncthreads();
  const int res = buf[warp] + __popc(m & ((1u << lane) - 1u));
  total = buf[kWarps];
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(kThreads, 1) topk_rows_kernel(const TopkParams P) {
  __shared__ int hist[2048];
  __shared__ int buf[kWarps + 1];
  __shared__ int pick_digit, pick_above;

  const int r = blockIdx.x;
  const int b = owner_seq(P.q_offsets, P.B, r);
  const int q0 = P.q_offsets[b];
  const int nq = P.q_offsets[b + 1] - q0;
  const int pos = P.ctx_lens[b] - nq + (r - q0);
  const int n = pos + 1;
  const int k = P.top_k;
  int32_t* const out = P.idx + static_cast<size_t>(r) * k;
  const float* const sc = P.scores + static_cast<size_t>(r) * P.ld;

  if (n <= k) {  // every causal position is kept
    for (int i = threadIdx.x; i < k; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }

  uint32_t prefix = 0, pmask = 0;
  int remaining = k;  // keys still to take at or below the current prefix
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass == 2 ? 0x3FFu : 0x7FFu;
    for (int i = threadIdx.x; i < 2048; i += kThreads) hist[i] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < n; s += kThreads) {
      const uint32_t key = score_key(sc[s]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1);
    }
    __syncthreads();
    // Thread t looks at digit pair u = 1023 - t, so the exclusive prefix in
    // thread order counts the keys in higher digits.
    const int u = kThreads - 1 - static_cast<int>(threadIdx.x);
    const int c_hi = hist[2 * u + 1], c_lo = hist[2 * u];
    int total;
    const int above = block_excl_sum(c_hi + c_lo, buf, total);
    if (above < remaining && remaining <= above + c_hi + c_lo) {
      if (above + c_hi >= remaining) {
        pick_digit = 2 * u + 1;
        pick_above = above;
      } else {
        pick_digit = 2 * u;
        pick_above = above + c_hi;
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(pick_digit) << shift;
    pmask |= dmask << shift;
    remaining -= pick_above;
    __syncthreads();
  }

  const uint32_t theta = prefix;
  const int need = remaining;  // keys equal to theta to keep, lowest positions first
  int taken_eq = 0, out_pos = 0;
#pragma unroll 1
  for (int base = 0; base < n && out_pos < k; base += kThreads) {
    const int s = base + static_cast<int>(threadIdx.x);
    const bool valid = s < n;
    const uint32_t key = valid ? score_key(sc[s]) : 0u;
    const bool gt = valid && key > theta;
    const bool eq = valid && key == theta;
    int eq_total, sel_total;
    const int eq_rank = taken_eq + block_excl_count(eq, buf, eq_total);
    const bool sel = gt || (eq && eq_rank < need);
    const int slot = out_pos + block_excl_count(sel, buf, sel_total);
    if (sel) out[slot] = s;
    taken_eq += eq_total;
    out_pos += sel_total;
  }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream) {
  if (a.Nq == 0) return cudaSuccess;
  TopkParams P;
  P.q_offsets = a.q_offsets;
  P.ctx_lens = a.ctx_lens;
  P.scores = a.scores;
  P.ld = a.ld;
  P.idx = a.idx;
  P.B = a.B;
  P.top_k = a.top_k;
  topk_rows_kernel<<<a.Nq, kThreads, 0, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace dsa
