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
// Launch shapes: many rows that fit one CTA's shared memory (a prefill) take
// one CTA per row, which finds the bin of the k-th key from a 12-bit
// histogram built while loading and runs the exact passes over that bin's
// keys only.  Few long rows (a standalone decode selection) take a
// thread-block cluster of 2-8 CTAs per row: each CTA holds a contiguous slice
// of the row's keys in shared memory, so the row is read from memory once;
// per-pass histograms are summed across the cluster through distributed
// shared memory (plain loads), and each CTA learns how many selections
// precede its slice from the other CTAs' counts.  Rows longer than 8 slices
// use the single-CTA kernel that re-reads the row each pass.  Decode inside
// the layer call uses the histogram path at the end of this file.
#include <cooperative_groups.h>

#include <algorithm>

#include "dsa_common.cuh"
#include "dsa_internal.h"
#include "select_common.cuh"

namespace cg = cooperative_groups;

namespace dsa {
namespace {

using namespace sel;

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
  const unsigned* err;  // an earlier kernel's error: skip the work
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

__global__ void __launch_bounds__(kThreads, 1) topk_rows_kernel(const TopkParams P) {
  __shared__ int hist[2048];
  __shared__ int buf[kWarps + 1];
  pdl_wait();
  pdl_launch_dependents();
  if (error_recorded(P.err)) return;  // nothing in this kernel sets it: uniform
  const int r = blockIdx.x;
  const int b = owner_seq(P.q_offsets, P.B, r);
  const int q0 = P.q_offsets[b];
  const int nq = P.q_offsets[b + 1] - q0;
  const int n = P.ctx_lens[b] - nq + (r - q0) + 1;
  const int k = P.top_k;
  int32_t* const out = P.idx + static_cast<size_t>(r) * k;
  if (n <= k) {  // every causal position is kept
    for (int i = threadIdx.x; i < k; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }
  row_select_global<kWarps>(P.scores + static_cast<size_t>(r) * P.ld, n, k, out, hist, buf);
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
  if (error_recorded(P.err)) return;  // the same for every CTA of the cluster
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


// ------------------------------------------------- histogram-driven path --
// For few long rows whose indexer launch built the score-key histograms.
constexpr int kHThreads = 512;
constexpr int kHWarps = kHThreads / 32;
constexpr int kCandMax = 8192;   // keys of the threshold bin kept for the exact pass
constexpr int kSortMax = 2048;   // >= top_k, power of two
constexpr int kFineBits = 11;    // sub-histogram of the threshold bin: the next 11 key bits
constexpr int kFineShift = kHistShift - kFineBits;
constexpr int kFineBins = 1 << kFineBits;

struct HistParams {
  const int32_t* q_offsets;
  const int32_t* ctx_lens;
  const float* scores;
  long long ld;
  int32_t* idx;
  int B, top_k, chunk, chunks;
  int* hist;            // [Nq][kHistBins], zeroed before the indexer runs
  int* fine;            // [Nq][kFineBins] sub-histogram of the threshold bin; zeroed too
  int* counters;        // [Nq][4]: keys above the bin, candidates, fallback flag; zeroed too
  uint32_t* cand_key;   // [Nq][kCandMax] keys of the threshold bin (any order)
  int* cand_pos;        // [Nq][kCandMax] their positions
  int* chunk_gt;        // [Nq][chunks][top_k] positions above the bin, per chunk
  int* chunk_ngt;       // [Nq][chunks] how many
  const unsigned* err;  // an earlier kernel's error: skip the work
};

// Finds, among `n` shared-memory keys, the `want`-th largest key theta and how
// many keys equal to theta are needed.  Every key has the bits `known_mask`
// equal to `known`; radix passes cover the bits in [lo_bit, hi_bit].  (The
// emit kernel's form, for 512 threads; the generic radix_select below,
// inlined there instead, made that kernel spill registers.)
__device__ void smem_select(const uint32_t* keys, int n, int want, int lo_bit, int hi_bit,
                            uint32_t known, uint32_t known_mask, int* hist /*[2048]*/, int* buf,
                            uint32_t& theta, int& need) {
  __shared__ int pd, pa;
  uint32_t prefix = known, pmask = known_mask;
  int remaining = want;
  for (int top = hi_bit; top >= lo_bit;) {
    const int nbits = min(11, top - lo_bit + 1);
    const int shift = top - nbits + 1;
    const uint32_t dmask = (1u << nbits) - 1u;
    for (int i = threadIdx.x; i < 2048; i += kHThreads) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kHThreads) {
      const uint32_t key = keys[i];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1);
    }
    __syncthreads();
    const int u = kHThreads - 1 - static_cast<int>(threadIdx.x);
    const int c0 = hist[4 * u], c1 = hist[4 * u + 1], c2 = hist[4 * u + 2], c3 = hist[4 * u + 3];
    const int tot = c0 + c1 + c2 + c3;
    int total;
    const int above = block_excl_sum_nw<kHWarps>(tot, buf, total);
    if (above < remaining && remaining <= above + tot) {
      if (above + c3 >= remaining) {
        pd = 4 * u + 3; pa = above;
      } else if (above + c3 + c2 >= remaining) {
        pd = 4 * u + 2; pa = above + c3;
      } else if (above + c3 + c2 + c1 >= remaining) {
        pd = 4 * u + 1; pa = above + c3 + c2;
      } else {
        pd = 4 * u; pa = above + c3 + c2 + c1;
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(pd) << shift;
    pmask |= dmask << shift;
    remaining -= pa;
    __syncthreads();
    top = shift - 1;
  }
  theta = prefix;
  need = remaining;
}

// Finds, among the `n` keys key_at(0 .. n-1), the `want`-th largest key theta
// and how many keys equal to theta are needed, with a block of kThr threads.
// Every key has the bits `known_mask` equal to `known`; radix passes of up to
// 11 bits cover the bits in [lo_bit, hi_bit].
template <int kThr, class KeyAt>
__device__ void radix_select(KeyAt key_at, int n, int want, int lo_bit, int hi_bit,
                             uint32_t known, uint32_t known_mask, int* hist /*[2048]*/, int* buf,
                             uint32_t& theta, int& need) {
  constexpr int kD = 2048 / kThr;  // digits per thread in the scan
  __shared__ int pd, pa;
  uint32_t prefix = known, pmask = known_mask;
  int remaining = want;
  for (int top = hi_bit; top >= lo_bit;) {
    const int nbits = min(11, top - lo_bit + 1);
    const int shift = top - nbits + 1;
    const uint32_t dmask = (1u << nbits) - 1u;
    for (int i = threadIdx.x; i < 2048; i += kThr) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kThr) {
      const uint32_t key = key_at(i);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1);
    }
    __syncthreads();
    // Thread t scans digits kD*u .. kD*u + kD-1 with u = kThr-1-t, so the
    // exclusive prefix in thread order counts the keys in higher digits.
    const int u = kThr - 1 - static_cast<int>(threadIdx.x);
    int c[kD];
    int tot = 0;
#pragma unroll
    for (int j = 0; j < kD; ++j) {
      c[j] = hist[kD * u + j];
      tot += c[j];
    }
    int total;
    int above = block_excl_sum_nw<kThr / 32>(tot, buf, total);
    if (above < remaining && remaining <= above + tot) {
#pragma unroll
      for (int j = kD - 1; j >= 0; --j) {
        if (above + c[j] >= remaining) {
          pd = kD * u + j;
          pa = above;
          break;
        }
        above += c[j];
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(pd) << shift;
    pmask |= dmask << shift;
    remaining -= pa;
    __syncthreads();
    top = shift - 1;
  }
  theta = prefix;
  need = remaining;
}

// ------------------------------------------------------- one CTA per row --
// Many rows (prefill): one 256-thread CTA per row.
//   1. count the keys by their top 12 bits (16-byte loads); one scan of the
//      4096 counts gives the bin holding the k-th largest key and how many
//      keys lie above it;
//   2. a second read of the row (from L2: it was just read) gives a bitmask
//      of the positions above that bin and a list of the keys inside it
//      (typically a few hundred) with their positions;
//   3. radix passes (11 + 9 bits) over the candidates alone give the k-th
//      key theta and how many keys equal to theta to keep; the selected
//      candidates are added to the bitmask (ties at theta: the lowest
//      positions, by a radix select on the complemented positions);
//   4. the positions are emitted in ascending order from the bitmask words,
//      placed by one block prefix sum of their bit counts.
// A bin holding more than kRowCandMax keys (heavy ties) takes the whole-row
// path instead: radix passes over every key of the row and an ordered
// emission, both re-reading the scores.
constexpr int kRowCandMax = 2048;
constexpr int kRThreads = 256;
constexpr int kRWarps = kRThreads / 32;

__device__ __forceinline__ void row_hist_add(int* hist, uint32_t key) {
  atomicAdd(&hist[key >> kHistShift], 1);
}

// Dynamic shared memory of the row kernel for rows of up to `slice` keys
// (a multiple of 128): histogram, candidates, bitmask.  Small enough that
// six rows share an SM, whose loads hide one another's latency.
__host__ __device__ constexpr size_t row_cta_smem(int slice) {
  return static_cast<size_t>(kHistBins) * sizeof(int) +
         static_cast<size_t>(kRowCandMax) * (sizeof(uint32_t) + sizeof(int)) +
         static_cast<size_t>(slice / 32) * sizeof(uint32_t);
}

__global__ void __launch_bounds__(kRThreads, 6) topk_row_cta_kernel(const TopkParams P) {
  extern __shared__ __align__(16) uint8_t smem[];
  int* const hist = reinterpret_cast<int*>(smem);                          // [kHistBins]
  uint32_t* const ckey = reinterpret_cast<uint32_t*>(hist + kHistBins);    // [kRowCandMax]
  int* const cpos = reinterpret_cast<int*>(ckey + kRowCandMax);            // [kRowCandMax]
  uint32_t* const mask = reinterpret_cast<uint32_t*>(cpos + kRowCandMax);  // [slice / 32]
  __shared__ int buf[kRWarps + 1];
  __shared__ int s_bin, s_above, s_cnt, s_ncand, s_neq;
  __shared__ int warp_gt[kRWarps], warp_eq[kRWarps];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_launch_dependents();
  if (error_recorded(P.err)) return;
  const int r = blockIdx.x;
  const int b = owner_seq(P.q_offsets, P.B, r);
  const int q0 = P.q_offsets[b];
  const int nq = P.q_offsets[b + 1] - q0;
  const int n = P.ctx_lens[b] - nq + (r - q0) + 1;  // positions 0..p; n <= slice
  const int k = P.top_k;
  int32_t* const out = P.idx + static_cast<size_t>(r) * k;
  if (n <= k) {  // every causal position is kept
    for (int i = tid; i < k; i += kRThreads) out[i] = i < n ? i : -1;
    return;
  }
  const float* const sc = P.scores + static_cast<size_t>(r) * P.ld;
  auto key_at = [&](int i) { return score_key(sc[i]); };

  // ---- sweep 1: coarse histogram
  for (int i = tid; i < kHistBins; i += kRThreads) hist[i] = 0;
  if (tid == 0) {
    s_ncand = 0;
    s_neq = 0;
  }
  if (tid < kRWarps) {
    warp_gt[tid] = 0;
    warp_eq[tid] = 0;
  }
  __syncthreads();
  const int n4 = (reinterpret_cast<uintptr_t>(sc) & 15u) == 0 ? (n & ~3) : 0;
  for (int i = 4 * tid; i < n4; i += 4 * kRThreads) {
    const float4 v = *reinterpret_cast<const float4*>(sc + i);
    row_hist_add(hist, score_key(v.x));
    row_hist_add(hist, score_key(v.y));
    row_hist_add(hist, score_key(v.z));
    row_hist_add(hist, score_key(v.w));
  }
  for (int i = n4 + tid; i < n; i += kRThreads) row_hist_add(hist, key_at(i));
  __syncthreads();
  {
    // Thread t holds bins 16u .. 16u+15 with u = 255 - t, so the exclusive
    // prefix in thread order counts the keys in higher bins.
    constexpr int kPer = kHistBins / kRThreads;
    const int u = kRThreads - 1 - tid;
    int c[kPer];
#pragma unroll
    for (int j = 0; j < kPer; j += 4) {
      const int4 h = reinterpret_cast<const int4*>(hist)[(kPer * u + j) / 4];
      c[j] = h.x;
      c[j + 1] = h.y;
      c[j + 2] = h.z;
      c[j + 3] = h.w;
    }
    int tot = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) tot += c[j];
    int total;
    int above = block_excl_sum_nw<kRWarps>(tot, buf, total);
    if (above < k && k <= above + tot) {
#pragma unroll
      for (int j = kPer - 1; j >= 0; --j) {
        if (above + c[j] >= k) {
          s_bin = kPer * u + j;
          s_above = above;
          s_cnt = c[j];
          break;
        }
        above += c[j];
      }
    }
  }
  __syncthreads();
  const int bin = s_bin;
  const int want = k - s_above;  // keys to keep from the bin, 1 .. s_cnt
  const uint32_t known = static_cast<uint32_t>(bin) << kHistShift;
  const uint32_t known_mask = ~((1u << kHistShift) - 1u);
  const unsigned lt = (1u << lane) - 1u;
  uint32_t theta;
  int need;

  if (s_cnt <= kRowCandMax) {
    // ---- sweep 2: bitmask above the bin, candidates
    const int W = (n + 31) >> 5;
    for (int w = warp; w < W; w += kRWarps) {
      const int i = 32 * w + lane;
      const uint32_t key = i < n ? key_at(i) : 0u;
      const int d = i < n ? static_cast<int>(key >> kHistShift) : -1;
      const unsigned gm = __ballot_sync(0xffffffffu, d > bin);
      const unsigned em = __ballot_sync(0xffffffffu, d == bin);
      if (lane == 0) mask[w] = gm;
      if (em != 0u) {
        int base = 0;
        if (lane == 0) base = atomicAdd(&s_ncand, __popc(em));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (d == bin) {
          const int j = base + __popc(em & lt);
          ckey[j] = key;
          cpos[j] = i;
        }
      }
    }
    __syncthreads();
    const int nc = s_ncand;
    radix_select<kRThreads>([&](int j) { return ckey[j]; }, nc, want, 0, kHistShift - 1, known,
                            known_mask, hist, buf, theta, need);
    // Keys equal to theta: keep the `need` lowest positions.
    for (int j = tid; j < nc; j += kRThreads) {
      if (ckey[j] == theta) atomicAdd(&s_neq, 1);
    }
    __syncthreads();
    uint32_t pos_cut = 0u;  // equal keys kept: ~position >= pos_cut
    if (need < s_neq) {
      int unused;
      radix_select<kRThreads>(
          [&](int j) { return ckey[j] == theta ? ~static_cast<uint32_t>(cpos[j]) : 0u; }, nc,
          need, 0, 31, 0u, 0u, hist, buf, pos_cut, unused);
    }
    for (int j = tid; j < nc; j += kRThreads) {
      const uint32_t key = ckey[j];
      const int pos = cpos[j];
      if (key > theta || (key == theta && ~static_cast<uint32_t>(pos) >= pos_cut)) {
        atomicOr(&mask[pos >> 5], 1u << (pos & 31));
      }
    }
    __syncthreads();
    // ---- emit from the bitmask: each thread a run of words, in order
    const int wpt = (W + kRThreads - 1) / kRThreads;
    const int wa = min(W, tid * wpt), wb = min(W, wa + wpt);
    int cnt = 0;
    for (int w = wa; w < wb; ++w) cnt += __popc(mask[w]);
    int total;
    int at = block_excl_sum_nw<kRWarps>(cnt, buf, total);
    for (int w = wa; w < wb; ++w) {
      uint32_t m = mask[w];
      while (m != 0u && at < k) {
        out[at++] = 32 * w + __ffs(m) - 1;
        m &= m - 1u;
      }
    }
    for (int i = total + tid; i < k; i += kRThreads) out[i] = -1;  // never with exact counts
    return;
  }

  // ---- heavy ties: radix passes over the whole row, then ordered emission
  const int per_warp = ((n + kRWarps - 1) / kRWarps + 31) & ~31;
  const int w0 = warp * per_warp;
  const int w1 = min(n, w0 + per_warp);
  radix_select<kRThreads>(key_at, n, want, 0, kHistShift - 1, known, known_mask, hist, buf, theta,
                          need);
  {
    int g = 0, e = 0;
    for (int i = w0 + lane; i < w0 + per_warp; i += 32) {
      const bool in = i < w1;
      const uint32_t key = in ? key_at(i) : 0u;
      g += __popc(__ballot_sync(0xffffffffu, in && key > theta));
      e += __popc(__ballot_sync(0xffffffffu, in && key == theta));
    }
    if (lane == 0) {
      warp_gt[warp] = g;
      warp_eq[warp] = e;
    }
  }
  __syncthreads();
  int eq_acc = 0, sel_acc = 0;
  for (int w = 0; w < warp; ++w) {
    sel_acc += warp_gt[w] + min(max(need - eq_acc, 0), warp_eq[w]);
    eq_acc += warp_eq[w];
  }
  for (int i = w0 + lane; i < w0 + per_warp; i += 32) {
    const bool in = i < w1;
    const uint32_t key = in ? key_at(i) : 0u;
    const unsigned gm = __ballot_sync(0xffffffffu, in && key > theta);
    const unsigned em = __ballot_sync(0xffffffffu, in && key == theta);
    const bool take_eq = ((em >> lane) & 1u) && eq_acc + __popc(em & lt) < need;
    const unsigned sm = gm | __ballot_sync(0xffffffffu, take_eq);
    if ((sm >> lane) & 1u) out[sel_acc + __popc(sm & lt)] = i;
    eq_acc += __popc(em);
    sel_acc += __popc(sm);
  }
}

// Row bookkeeping shared by the two kernels of the histogram path.
struct HistRow {
  int r, c;
  int* gh;
  int* cnt;
  int32_t* out;
  const float* sc;
};

__device__ __forceinline__ HistRow hist_row(const HistParams& P) {
  HistRow h;
  h.r = blockIdx.x / P.chunks;
  h.c = blockIdx.x - h.r * P.chunks;
  h.gh = P.hist + static_cast<size_t>(h.r) * kHistBins;
  h.cnt = P.counters + static_cast<size_t>(h.r) * 4;
  h.out = P.idx + static_cast<size_t>(h.r) * P.top_k;
  h.sc = P.scores + static_cast<size_t>(h.r) * P.ld;
  return h;
}

// Causal length of query row r, looked up by one warp with all of its loads
// in flight at once (lane l checks sequences l, l + 32, ...).
__device__ __forceinline__ int row_causal_len_warp(const HistParams& P, int r) {
  int n = 0;
  for (int b = threadIdx.x & 31; b < P.B; b += 32) {
    const int q0 = __ldg(P.q_offsets + b), q1 = __ldg(P.q_offsets + b + 1);
    const int L = __ldg(P.ctx_lens + b);
    if (r >= q0 && r < q1) n = L - (q1 - q0) + (r - q0) + 1;
  }
  return __reduce_max_sync(0xffffffffu, n);
}

// Filter: the bin holding the k-th largest key comes from the histogram the
// indexer built; one pass over this CTA's chunk keeps the positions above
// the bin (per chunk, for the emit kernel) and the keys in the bin (the
// row's candidates), and counts the candidates by the next kFineBits key
// bits into the row's sub-histogram.
__global__ void __launch_bounds__(kHThreads, 2) topk_filter_kernel(const HistParams P) {
  extern __shared__ __align__(16) uint8_t hsm[];
  int* const st_gt = reinterpret_cast<int*>(hsm);                         // [kSortMax]
  uint32_t* const st_ck = reinterpret_cast<uint32_t*>(st_gt + kSortMax);  // [kCandMax]
  int* const st_cp = reinterpret_cast<int*>(st_ck + kCandMax);            // [kCandMax]
  __shared__ int buf[kHWarps + 1];
  __shared__ int s_bin, s_above, s_inbin, s_ngt, s_nc, s_cbase;

  pdl_wait();
  pdl_launch_dependents();
  if (error_recorded(P.err)) return;
  const int tid = threadIdx.x, lane = tid & 31;
  const HistRow R = hist_row(P);
  const int k = P.top_k;
  __shared__ int s_n;
  if (tid < 32) {  // the row's length, while the other warps' loads go out
    const int n = row_causal_len_warp(P, R.r);
    if (tid == 0) s_n = n;
  }
  // The chunk's scores (within the row's stride; masked by the length below)
  // and the row's histogram are loaded before anything waits on them.
  const int s0 = R.c * P.chunk;
  const int s_end = static_cast<int>(min(static_cast<long long>(s0 + P.chunk), P.ld));
  constexpr int kPer = kCandMax / kHThreads;
  uint32_t keys[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int s = s0 + j * kHThreads + tid;
    keys[j] = s < s_end ? score_key(__ldcg(R.sc + s)) : 0u;
  }
  const int u = kHThreads - 1 - tid;  // thread t reads bins 8u .. 8u+7, u = 511 - t
  // Two 16-byte loads per thread: every CTA of the row reads this histogram.
  const int4 h0 = __ldcg(reinterpret_cast<const int4*>(R.gh) + 2 * u);
  const int4 h1 = __ldcg(reinterpret_cast<const int4*>(R.gh) + 2 * u + 1);
  const int cb[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  int tot = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) tot += cb[j];
  __syncthreads();
  const int n = s_n;
  if (R.c == 0 && tid == 0) R.cnt[3] = n;
  if (n <= k) {  // every causal position is kept
    if (R.c == 0) {
      for (int i = tid; i < k; i += kHThreads) R.out[i] = i < n ? i : -1;
    }
    return;
  }
  if (s0 >= n) return;  // chunk past the row's end (chunk 0 never is)
  const int s1 = min(n, s0 + P.chunk);
  // The bin of the k-th largest key: the prefix in thread order counts the
  // keys in higher bins.
  {
    int total;
    int above = block_excl_sum_nw<kHWarps>(tot, buf, total);
    if (above < k && k <= above + tot) {
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        if (above + cb[j] >= k) {
          s_bin = 8 * u + j;
          s_above = above;
          s_inbin = cb[j];
          break;
        }
        above += cb[j];
      }
    }
    if (tid == 0) {
      s_ngt = 0;
      s_nc = 0;
    }
    __syncthreads();
  }
  const uint32_t bstar = static_cast<uint32_t>(s_bin);
  const int c_above = s_above, c_in = s_inbin;
  if (R.c == 0 && tid == 0) {
    R.cnt[0] = c_above;
    R.cnt[2] = c_in > kCandMax;  // too many keys in the bin: whole-row fallback
  }
  if (c_in > kCandMax) return;

  const unsigned lt = (1u << lane) - 1u;
  int* const fine = P.fine + static_cast<size_t>(R.r) * kFineBins;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    if (s0 + j * kHThreads >= s1) break;
    const int s = s0 + j * kHThreads + tid;
    const bool in = s < s1;
    const uint32_t bin = keys[j] >> kHistShift;
    const bool gt = in && bin > bstar;
    const bool eq = in && bin == bstar;
    const unsigned mg = __ballot_sync(0xffffffffu, gt);
    const unsigned me = __ballot_sync(0xffffffffu, eq);
    if (mg) {
      int at = 0;
      if (lane == 0) at = atomicAdd(&s_ngt, __popc(mg));
      at = __shfl_sync(0xffffffffu, at, 0) + __popc(mg & lt);
      if (gt && at < kSortMax) st_gt[at] = s;
    }
    if (me) {
      int at = 0;
      if (lane == 0) at = atomicAdd(&s_nc, __popc(me));
      at = __shfl_sync(0xffffffffu, at, 0) + __popc(me & lt);
      if (eq) {
        atomicAdd(fine + ((keys[j] >> kFineShift) & (kFineBins - 1)), 1);
        if (at < kCandMax) {
          st_ck[at] = keys[j];
          st_cp[at] = s;
        }
      }
    }
  }
  __syncthreads();
  if (tid == 0) s_cbase = atomicAdd(&R.cnt[1], s_nc);
  __syncthreads();
  const int ngt = min(s_ngt, k);
  int* const cg = P.chunk_gt + (static_cast<size_t>(R.r) * P.chunks + R.c) * k;
  for (int i = tid; i < ngt; i += kHThreads) cg[i] = st_gt[i];
  if (tid == 0) P.chunk_ngt[static_cast<size_t>(R.r) * P.chunks + R.c] = ngt;
  for (int i = tid; i < s_nc; i += kHThreads) {
    const int slot = s_cbase + i;
    if (slot < kCandMax) {
      P.cand_key[static_cast<size_t>(R.r) * kCandMax + slot] = st_ck[i];
      P.cand_pos[static_cast<size_t>(R.r) * kCandMax + slot] = st_cp[i];
    }
  }
}

// Emit: from the row's sub-histogram every CTA of the row finds the sub-bin
// holding the k-th largest key (the same, redundantly, in parallel) and
// ranks the few candidates inside it exactly (score desc, position asc);
// then it counts the selected candidates of earlier chunks and writes its
// own chunk's selected positions, sorted, after those of earlier chunks.
constexpr int kMaxChunks = 512;
constexpr int kMemberMax = 2048;  // keys of the sub-bin ranked in shared memory
constexpr int kRankDirect = 64;   // up to this many, by pairwise comparison
__global__ void __launch_bounds__(kHThreads, 2) topk_emit_kernel(const HistParams P) {
  __shared__ uint32_t mk[kMemberMax];  // sub-bin keys
  __shared__ int mp[kMemberMax];       // their positions
  __shared__ uint32_t tk[kMemberMax];  // tie keys for the position cut
  __shared__ uint8_t mkeep[kMemberMax];
  __shared__ int fin[kSortMax];        // this chunk's selected positions
  __shared__ int hist[2048];
  __shared__ int buf[kHWarps + 1];
  __shared__ int s_b2, s_above2, s_c2, s_nm, s_nown;

  pdl_wait();
  pdl_launch_dependents();
  if (error_recorded(P.err)) return;
  const int tid = threadIdx.x;
  const HistRow R = hist_row(P);
  const int k = P.top_k;
  // Everything the first decisions need, loaded at once: the row's counters
  // (keys above the bin, candidates, fallback flag, causal length), the
  // per-chunk counts of positions above the bin, and the sub-histogram.
  const int4 cn = __ldcg(reinterpret_cast<const int4*>(R.cnt));
  const int* const ngt = P.chunk_ngt + static_cast<size_t>(R.r) * P.chunks;
  const int own_gt_raw = __ldcg(ngt + R.c);
  int gt_before = tid < R.c ? __ldcg(ngt + tid) : 0;  // chunks <= kMaxChunks = threads
  const int4 f = __ldcg(reinterpret_cast<const int4*>(P.fine + static_cast<size_t>(R.r) *
                                                                   kFineBins) +
                        (kHThreads - 1 - tid));
  const int c_above = cn.x, c_in = cn.y, fallback = cn.z, n = cn.w;
  if (n <= k || R.c * P.chunk >= n) return;
  if (fallback != 0) {  // heavily tied scores: whole-row selection by one CTA
    if (R.c == 0) row_select_global<kHWarps>(R.sc, n, k, R.out, hist, buf);
    return;
  }
  const int own_gt = min(own_gt_raw, k);
  constexpr int kPer = kCandMax / kHThreads;
  uint32_t ck[kPer];
  int cp[kPer];
  const uint32_t* const gk = P.cand_key + static_cast<size_t>(R.r) * kCandMax;
  const int* const gp = P.cand_pos + static_cast<size_t>(R.r) * kCandMax;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = j * kHThreads + tid;
    ck[j] = i < c_in ? __ldcg(gk + i) : 0u;
    cp[j] = i < c_in ? __ldcg(gp + i) : 0;
  }
  const int* const cg = P.chunk_gt + (static_cast<size_t>(R.r) * P.chunks + R.c) * k;
  const int gt_mine = tid < own_gt ? __ldcg(cg + tid) : 0;  // the first two of up to four rounds
  const int gt_mine2 = tid + kHThreads < own_gt ? __ldcg(cg + tid + kHThreads) : 0;
  // Sub-bin of the k-th largest key; thread t reads sub-bins 4u .. 4u+3, u = 511 - t.
  const int need = k - c_above;  // candidates to keep, 1 <= need <= c_in
  {
    const int tot = f.x + f.y + f.z + f.w;
    int total;
    const int above = block_excl_sum_nw<kHWarps>(tot, buf, total);
    const int u = kHThreads - 1 - tid;
    if (above < need && need <= above + tot) {
      if (above + f.w >= need) {
        s_b2 = 4 * u + 3; s_above2 = above; s_c2 = f.w;
      } else if (above + f.w + f.z >= need) {
        s_b2 = 4 * u + 2; s_above2 = above + f.w; s_c2 = f.z;
      } else if (above + f.w + f.z + f.y >= need) {
        s_b2 = 4 * u + 1; s_above2 = above + f.w + f.z; s_c2 = f.y;
      } else {
        s_b2 = 4 * u; s_above2 = above + f.w + f.z + f.y; s_c2 = f.x;
      }
    }
    if (tid == 0) {
      s_nm = 0;
      s_nown = 0;
    }
    __syncthreads();
  }
  const uint32_t b2 = static_cast<uint32_t>(s_b2);
  const int need2 = need - s_above2;  // members of the sub-bin to keep, 1 <= need2 <= c2
  if (s_c2 > kMemberMax) {            // every CTA of the row sees the same count
    if (R.c == 0) row_select_global<kHWarps>(R.sc, n, k, R.out, hist, buf);
    return;
  }
  const int lo = R.c * P.chunk, hi = lo + P.chunk;
  int before = gt_before;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    if (j * kHThreads >= c_in) break;
    if (j * kHThreads + tid >= c_in) continue;
    const uint32_t sub = (ck[j] >> kFineShift) & (kFineBins - 1);
    if (sub > b2) {
      before += cp[j] < lo;
      if (cp[j] >= lo && cp[j] < hi) {
        const int at = atomicAdd(&s_nown, 1);
        if (at < kSortMax) fin[at] = cp[j];
      }
    } else if (sub == b2) {
      const int at = atomicAdd(&s_nm, 1);
      if (at < kMemberMax) {
        mk[at] = ck[j];
        mp[at] = cp[j];
      }
    }
  }
  __syncthreads();
  const int nm = min(s_nm, kMemberMax);  // == c2
  if (need2 >= nm) {
    for (int i = tid; i < nm; i += kHThreads) mkeep[i] = 1;
  } else if (nm <= kRankDirect) {
    for (int i = tid; i < nm; i += kHThreads) {
      int rank = 0;
      for (int j = 0; j < nm; ++j) {
        rank += mk[j] > mk[i] || (mk[j] == mk[i] && mp[j] < mp[i]);
      }
      mkeep[i] = rank < need2;
    }
  } else {
    const uint32_t known_mask = ~((1u << kFineShift) - 1u);
    uint32_t theta;
    int need_eq;
    smem_select(mk, nm, need2, 0, kFineShift - 1, mk[0] & known_mask, known_mask, hist, buf,
                theta, need_eq);
    int n_tie = 0;
    for (int i = tid; i < nm; i += kHThreads) n_tie += mk[i] == theta;
    int total_tie;
    block_excl_sum_nw<kHWarps>(n_tie, buf, total_tie);
    uint32_t pos_cut = 0u;  // ties kept: ~position >= pos_cut (the lowest positions)
    const bool cut_ties = need_eq < total_tie;
    if (cut_ties) {
      for (int i = tid; i < nm; i += kHThreads) {
        tk[i] = mk[i] == theta ? ~static_cast<uint32_t>(mp[i]) : 0u;
      }
      __syncthreads();
      int unique;
      smem_select(tk, nm, need_eq, 0, 31, 0u, 0u, hist, buf, pos_cut, unique);
    }
    for (int i = tid; i < nm; i += kHThreads) {
      mkeep[i] = mk[i] > theta ||
                 (mk[i] == theta && (!cut_ties || ~static_cast<uint32_t>(mp[i]) >= pos_cut));
    }
  }
  __syncthreads();
  for (int i = tid; i < nm; i += kHThreads) {
    if (mkeep[i]) {
      before += mp[i] < lo;
      if (mp[i] >= lo && mp[i] < hi) {
        const int at = atomicAdd(&s_nown, 1);
        if (at < kSortMax) fin[at] = mp[i];
      }
    }
  }
  int offset;
  block_excl_sum_nw<kHWarps>(before, buf, offset);  // total: selections in earlier chunks
  const int n_cand_own = min(s_nown, kSortMax);
  const int m = min(n_cand_own + own_gt, kSortMax);
  if (tid + n_cand_own < m) fin[n_cand_own + tid] = gt_mine;
  if (tid + kHThreads + n_cand_own < m) fin[n_cand_own + kHThreads + tid] = gt_mine2;
  for (int i = tid + 2 * kHThreads; i + n_cand_own < m; i += kHThreads) {
    fin[n_cand_own + i] = __ldcg(cg + i);
  }
  __syncthreads();
  if (m <= 64) {  // the usual case: one warp sorts two positions per lane with shuffles
    if (tid < 32) {
      int v0 = tid < m ? fin[tid] : 0x7FFFFFFF;
      int v1 = tid + 32 < m ? fin[tid + 32] : 0x7FFFFFFF;
#pragma unroll
      for (int sz = 2; sz <= 64; sz <<= 1) {  // ascending bitonic network over 64 slots
#pragma unroll
        for (int stride = sz >> 1; stride > 0; stride >>= 1) {
          if (stride == 32) {  // slots tid and tid + 32 of this lane (sz = 64: ascending)
            const int lo_v = min(v0, v1), hi_v = max(v0, v1);
            v0 = lo_v;
            v1 = hi_v;
          } else {
            const bool lower = (tid & stride) == 0;
            const int p0 = __shfl_xor_sync(0xffffffffu, v0, stride);
            const int p1 = __shfl_xor_sync(0xffffffffu, v1, stride);
            const bool up0 = (tid & sz) == 0, up1 = ((tid + 32) & sz) == 0;
            v0 = (lower == up0) ? min(v0, p0) : max(v0, p0);
            v1 = (lower == up1) ? min(v1, p1) : max(v1, p1);
          }
        }
      }
      if (tid < m && offset + tid < k) R.out[offset + tid] = v0;
      if (tid + 32 < m && offset + tid + 32 < k) R.out[offset + tid + 32] = v1;
    }
    return;
  }
  int size = 1;
  while (size < m) size <<= 1;
  for (int i = m + tid; i < size; i += kHThreads) fin[i] = 0x7FFFFFFF;
  __syncthreads();
  for (int sz = 2; sz <= size; sz <<= 1) {  // ascending bitonic sort of the m positions
    for (int stride = sz >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < size; i += kHThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const int a = fin[i], bb = fin[j];
          const bool up = (i & sz) == 0;
          if ((a > bb) == up) {
            fin[i] = bb;
            fin[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < m; i += kHThreads) {
    if (offset + i < k) R.out[offset + i] = fin[i];
  }
}

}  // namespace

int topk_hist_chunks(int Nq, int64_t max_len, int* chunk_len) {
  // About two CTAs per SM of a 148-SM part in all, chunks of whole 512-key
  // blocks, at most kCandMax keys (the shared staging arrays) per chunk.
  int chunks = std::max(1, 2 * 148 / std::max(1, Nq));
  int chunk = static_cast<int>(((max_len + chunks - 1) / chunks + kHThreads - 1) / kHThreads *
                               kHThreads);
  chunk = std::max(kHThreads, std::min(chunk, kCandMax));
  chunks = static_cast<int>((max_len + chunk - 1) / chunk);
  if (chunk_len) *chunk_len = chunk;
  return chunks;
}

bool topk_hist_supported(int Nq, int64_t max_len) {
  return topk_hist_chunks(Nq, max_len, nullptr) <= kMaxChunks;
}

size_t topk_hist_zero_bytes(int Nq) {
  return static_cast<size_t>(Nq) * (kHistBins + kFineBins + 4) * sizeof(int);
}

size_t topk_hist_ws_bytes(int Nq, int top_k, int64_t max_len) {
  const int chunks = topk_hist_chunks(Nq, max_len, nullptr);
  return topk_hist_zero_bytes(Nq) +
         static_cast<size_t>(Nq) * (kCandMax * (sizeof(uint32_t) + sizeof(int))) +
         static_cast<size_t>(Nq) * chunks * (static_cast<size_t>(top_k) + 1) * sizeof(int);
}

cudaError_t launch_topk_hist(const TopkArgs& a, void* ws_region, cudaStream_t stream) {
  if (a.Nq == 0) return cudaSuccess;
  HistParams P;
  P.q_offsets = a.q_offsets;
  P.ctx_lens = a.ctx_lens;
  P.scores = a.scores;
  P.ld = a.ld;
  P.idx = a.idx;
  P.B = a.B;
  P.top_k = a.top_k;
  P.err = a.err;
  P.chunks = topk_hist_chunks(a.Nq, a.max_len, &P.chunk);
  uint8_t* p = static_cast<uint8_t*>(ws_region);
  P.hist = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(a.Nq) * kHistBins * sizeof(int);
  P.fine = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(a.Nq) * kFineBins * sizeof(int);
  P.counters = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(a.Nq) * 4 * sizeof(int);
  P.cand_key = reinterpret_cast<uint32_t*>(p);
  p += static_cast<size_t>(a.Nq) * kCandMax * sizeof(uint32_t);
  P.cand_pos = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(a.Nq) * kCandMax * sizeof(int);
  P.chunk_gt = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(a.Nq) * P.chunks * a.top_k * sizeof(int);
  P.chunk_ngt = reinterpret_cast<int*>(p);
  const size_t smem_f = static_cast<size_t>(kSortMax) * 4 + static_cast<size_t>(kCandMax) * 8;
  cudaError_t e = ensure_smem_limit<topk_filter_kernel>(static_cast<int>(smem_f));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(a.Nq) * P.chunks);
  e = launch_pdl(topk_filter_kernel, grid, dim3(kHThreads), smem_f, stream, 0, P);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_emit_kernel, grid, dim3(kHThreads), 0, stream, 0, P);
}

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
  P.err = a.err;
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
  if (cs == 1) {  // many rows, one CTA each
    // The limit is raised once, to the largest slice any launch may use.
    cudaError_t e = ensure_smem_limit<topk_row_cta_kernel>(static_cast<int>(row_cta_smem(kMaxSlice)));
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_row_cta_kernel, dim3(static_cast<unsigned>(a.Nq)), dim3(kRThreads),
                      row_cta_smem(P.slice), stream, 0, P);
  }
  const size_t smem = 2 * kBins * sizeof(int) + static_cast<size_t>(P.slice) * sizeof(uint32_t);
  // The limit is raised once, to the largest slice any launch may use.
  cudaError_t e = ensure_smem_limit<topk_cluster_kernel>(
      static_cast<int>(2 * kBins * sizeof(int) + static_cast<size_t>(kMaxSlice) * sizeof(uint32_t)));
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_cluster_kernel, dim3(static_cast<unsigned>(a.Nq) * cs), dim3(kCThreads),
                    smem, stream, cs, P);
}

}  // namespace dsa
