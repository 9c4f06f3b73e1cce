// Top-k token selection per query row.
//
// Keeps the n = min(top_k, p+1) positions of 0..p with the largest
// (score, -position): score descending, ties to the lower position
// (llama.cpp b12180 news: aiaulis.com paragraphs 2-3 — only the
// highest-scored tokens are attended, 2048 of them; devotd.net configuration
// table).  Output is in ascending position order, padded with -1.
//
// Method: scores are mapped to order-preserving uint32 keys; a three-pass MSB
// radix select (11 + 11 + 10 bits) finds the exact k-th largest key theta and
// how many of the keys equal to theta are needed; an ordered pass emits every
// key > theta plus the first `need` keys == theta, compacting with ballot
// prefix counts so the output is deterministic and sorted by position.
//
// Main kernel: a thread-block cluster of CS CTAs per row (CS = 1 for the many
// short rows of a prefill, up to 8 for the few long rows of a decode).  Each
// CTA holds a contiguous slice of the row's keys in shared memory, so the row
// is read from memory once; per-pass histograms are summed across the cluster
// through distributed shared memory (plain loads), and each CTA learns how
// many selections precede its slice from the other CTAs' counts.  Rows longer
// than 8 slices use the single-CTA kernel that re-reads the row each pass.
#include <cooperative_groups.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace cg = cooperative_groups;

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

constexpr int kCThreads = 512;   // cluster kernel
constexpr int kCWarps = kCThreads / 32;
constexpr int kBins = 2048;
constexpr int kMaxCluster = 8;
constexpr int kMaxSlice = 49152;  // keys per CTA (192 KB of shared memory)

struct TopkParams {
  const int32_t* q_offsets;
  const int32_t* ctx_lens;
  const float* scores;
  long long ld;
  int32_t* idx;
  int B;
  int top_k;
  int slice;  // keys per CTA (cluster kernel)
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

  pdl_wait();
  pdl_launch_dependents();
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

__global__ void __launch_bounds__(kCThreads) topk_cluster_kernel(const TopkParams P) {
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) uint8_t smem[];
  int* const hist = reinterpret_cast<int*>(smem);                       // [2][kBins]
  uint32_t* const keys = reinterpret_cast<uint32_t*>(hist + 2 * kBins);  // [slice]
  __shared__ int buf[kCWarps + 1];
  __shared__ int pick_digit, pick_above;
  __shared__ int slice_cnt[2];  // keys > theta and keys == theta in this slice
  __shared__ int warp_gt[kCWarps], warp_eq[kCWarps];

  const int CS = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_launch_dependents();
  const int r = blockIdx.x / CS;
  const int b = owner_seq(P.q_offsets, P.B, r);
  const int q0 = P.q_offsets[b];
  const int nq = P.q_offsets[b + 1] - q0;
  const int n = P.ctx_lens[b] - nq + (r - q0) + 1;  // positions 0..p
  const int k = P.top_k;
  int32_t* const out = P.idx + static_cast<size_t>(r) * k;

  if (n <= k) {  // the whole cluster leaves together: every causal position is kept
    if (rank == 0) {
      for (int i = tid; i < k; i += kCThreads) out[i] = i < n ? i : -1;
    }
    return;
  }

  const int s0 = rank * P.slice;
  const int len = max(0, min(n - s0, P.slice));
  const float* const sc = P.scores + static_cast<size_t>(r) * P.ld + s0;
  for (int i = tid; i < len; i += kCThreads) keys[i] = score_key(sc[i]);

  uint32_t prefix = 0, pmask = 0;
  int remaining = k;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass == 2 ? 0x3FFu : 0x7FFu;
    // Double-buffered: every CTA finished reading this buffer (two passes ago)
    // before it arrived at the previous cluster barrier.
    int* const h = hist + (pass & 1) * kBins;
    for (int i = tid; i < kBins; i += kCThreads) h[i] = 0;
    __syncthreads();
    for (int base = 0; base < len; base += kCThreads) {
      const int i = base + tid;
      const uint32_t key = i < len ? keys[i] : 0u;
      const bool v = i < len && (key & pmask) == prefix;
      const uint32_t bin = v ? (key >> shift) & dmask : 0xFFFFFFFFu;
      const unsigned grp = __match_any_sync(0xffffffffu, bin);
      if (v && lane == __ffs(grp) - 1) atomicAdd(&h[bin], __popc(grp));
    }
    cluster.sync();
    // Cluster totals of digits 4u .. 4u+3; thread order runs from the top digit down.
    const int u = kCThreads - 1 - tid;
    int c0 = 0, c1 = 0, c2 = 0, c3 = 0;
    for (int q = 0; q < CS; ++q) {
      const int4 x = reinterpret_cast<const int4*>(cluster.map_shared_rank(h, q))[u];
      c0 += x.x;
      c1 += x.y;
      c2 += x.z;
      c3 += x.w;
    }
    const int tot = c0 + c1 + c2 + c3;
    int total;
    const int above = block_excl_sum_nw<kCWarps>(tot, buf, total);
    if (above < remaining && remaining <= above + tot) {
      if (above + c3 >= remaining) {
        pick_digit = 4 * u + 3;
        pick_above = above;
      } else if (above + c3 + c2 >= remaining) {
        pick_digit = 4 * u + 2;
        pick_above = above + c3;
      } else if (above + c3 + c2 + c1 >= remaining) {
        pick_digit = 4 * u + 1;
        pick_above = above + c3 + c2;
      } else {
        pick_digit = 4 * u;
        pick_above = above + c3 + c2 + c1;
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(pick_digit) << shift;
    pmask |= dmask << shift;
    remaining -= pick_above;
  }

  const uint32_t theta = prefix;
  const int need = remaining;  // keys equal to theta to keep, lowest positions first
  // Each warp owns a contiguous chunk of the slice; count its > and == keys.
  const int per_warp = ((len + kCWarps - 1) / kCWarps + 31) & ~31;
  const int w0 = warp * per_warp;
  const int w1 = min(len, w0 + per_warp);
  int g = 0, e = 0;
  for (int i = w0 + lane; i < w0 + per_warp; i += 32) {
    const bool in = i < w1;
    const uint32_t key = in ? keys[i] : 0u;
    g += __popc(__ballot_sync(0xffffffffu, in && key > theta));
    e += __popc(__ballot_sync(0xffffffffu, in && key == theta));
  }
  if (lane == 0) {
    warp_gt[warp] = g;
    warp_eq[warp] = e;
  }
  __syncthreads();
  if (tid == 0) {
    int sg = 0, se = 0;
    for (int w = 0; w < kCWarps; ++w) {
      sg += warp_gt[w];
      se += warp_eq[w];
    }
    slice_cnt[0] = sg;
    slice_cnt[1] = se;
  }
  cluster.sync();
  // Selections and ties that precede this slice (lower ranks hold lower positions).
  int eq_acc = 0, sel_acc = 0;
  for (int q = 0; q < rank; ++q) {
    const int* rc = cluster.map_shared_rank(slice_cnt, q);
    const int gq = rc[0], eqq = rc[1];
    sel_acc += gq + min(max(need - eq_acc, 0), eqq);
    eq_acc += eqq;
  }
  cluster.sync();  // no CTA leaves while another still reads its counts
  for (int w = 0; w < warp; ++w) {
    sel_acc += warp_gt[w] + min(max(need - eq_acc, 0), warp_eq[w]);
    eq_acc += warp_eq[w];
  }
  const unsigned lt = (1u << lane) - 1u;
  for (int i = w0 + lane; i < w0 + per_warp; i += 32) {
    const bool in = i < w1;
    const uint32_t key = in ? keys[i] : 0u;
    const unsigned gm = __ballot_sync(0xffffffffu, in && key > theta);
    const unsigned em = __ballot_sync(0xffffffffu, in && key == theta);
    const bool take_eq = ((em >> lane) & 1u) && eq_acc + __popc(em & lt) < need;
    const unsigned sm = gm | __ballot_sync(0xffffffffu, take_eq);
    if ((sm >> lane) & 1u) out[sel_acc + __popc(sm & lt)] = s0 + i;
    eq_acc += __popc(em);
    sel_acc += __popc(sm);
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
  P.slice = 0;
  const long long n_max = a.max_len;
  auto slice_of = [&](int cs) { return static_cast<long long>((n_max + cs - 1) / cs + 127) / 128 * 128; };
  // Cluster size: enough CTAs for the row to fit, more while the GPU has idle
  // SMs and slices stay above 4096 keys.
  int cs = 1;
  while (cs < kMaxCluster &&
         (slice_of(cs) > kMaxSlice ||
          (2LL * a.Nq * cs <= a.num_sms && slice_of(cs) > 4096))) {
    cs *= 2;
  }
  if (slice_of(cs) > kMaxSlice) {  // longer than the cluster can hold
    P.slice = 0;
    return launch_pdl(topk_rows_kernel, dim3(a.Nq), dim3(kThreads), 0, stream, 0, P);
  }
  P.slice = static_cast<int>(slice_of(cs));
  const size_t smem = 2 * kBins * sizeof(int) + static_cast<size_t>(P.slice) * sizeof(uint32_t);
  // The limit is raised once, to the largest slice any launch may use.
  cudaError_t e = ensure_smem_limit<topk_cluster_kernel>(
      static_cast<int>(2 * kBins * sizeof(int) + static_cast<size_t>(kMaxSlice) * sizeof(uint32_t)));
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_cluster_kernel, dim3(static_cast<unsigned>(a.Nq) * cs), dim3(kCThreads),
                    smem, stream, cs, P);
}

}  // namespace dsa
