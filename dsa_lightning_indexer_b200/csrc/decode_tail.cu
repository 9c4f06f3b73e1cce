// The decode layer after the indexer, as one kernel: top-k selection driven
// by the indexer's score histograms, attention over the selected latent rows
// on tcgen05 tensor cores, and the merge of the row's partial results.
//
//   S_q = the min(top_k, p+1) positions of 0..p with the largest (score, -pos)
//   O[q, g, :] = sum_{s in S_q} softmax_s(scale * q[q, g, :] . kv[s, :]) * kv[s, :512]
//
// (llama.cpp b12180 news: aiaulis.com paragraphs 2-3 -- attention only over
// the highest-scored tokens, 2048 of them; devotd.net section 2 -- one
// key-only latent cache whose leading 512 entries serve as V.)
//
// One cooperative launch of Nq x C CTAs (one per SM); CTA (r, c) owns chunk
// c of row r's causal positions [s0, s1).  Phases:
//   A  From the row's 4096-bin histogram of the top 12 key bits (built by the
//      indexer) find the bin holding the k-th largest key.  Read the chunk's
//      scores once: positions above that bin are selected for sure, positions
//      in it are candidates (appended to the row's candidate list and counted
//      into the row's 2048-bin sub-histogram of the next 11 key bits).  The
//      latent rows of both start coming into L2; then arrive on the row's
//      counter.
//   B  When every CTA of the row has arrived, find the sub-bin of the k-th
//      key and rank its few members exactly; write this chunk's selected
//      positions, in order, into the row's index set.  Heavily tied rows
//      (candidate list or sub-bin too full) fall back to an exact whole-row
//      select by the row's first CTA.
//   C  Attend over the chunk's own selected positions when every chunk of
//      the row holds at most one tile of them (known to every CTA from the
//      per-chunk counts, so no further barrier); otherwise, once the index
//      set is complete, over slots [c*ceil(k/C), ...) of it.  Rows are
//      gathered in tiles of 96: S = Q K^T, softmax, P as bf16 hi + lo,
//      O^T = V^T P^T into TMEM with a running maximum; the unnormalised O
//      and (max, sum) of every head go to the row's partial results.
//   D  When every CTA of the row has stored its partials, each merges a
//      1/C share of the row's output with the log-sum-exp rule.
// Every wait is bounded; a wait that runs out sets the workspace error word
// and the CTA skips to its exit, after its own copies and MMAs have drained.
#include <algorithm>

#include "attn_tc_common.cuh"
#include "select_common.cuh"

namespace dsa {
namespace {

using namespace attn_tc;
using namespace sel;

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kTile = 96;                 // gathered rows per tile
constexpr int kHB = 64;                   // heads per CTA (H <= 64)
constexpr int kBoxes = kLatent / 64;
constexpr int kQBox = kHB * 128;
constexpr int kKVBox = kTile * 128;
constexpr int kPBlk = kHB * 128;          // P^T block: 64 heads x 64 keys bf16
constexpr int kMaxWords = 512;            // chunk <= 16384 positions
constexpr int kWordsPerWarp = 8;          // 32-position words per warp per pass (16 warps)
constexpr int kCandMax = 8192;            // candidates kept per row
constexpr int kCandPer = 4;               // candidates per thread per batch in phase B
constexpr int kMemberMax = 512;           // sub-bin members ranked in shared memory
constexpr int kFineBits = 11;
constexpr int kFineShift = kHistShift - kFineBits;
constexpr int kFineBins = 1 << kFineBits;
constexpr int kHalf = kTile / 2;          // logits per half warp
constexpr int kSoftThreads = 128;
constexpr float kRescaleLog2 = 0.0f;      // raise the running max whenever it grows

// Per-row counters (int): candidates appended, arrivals after phase A,
// arrivals after the partials, arrivals after the index set is written.
constexpr int kCtrCand = 0, kCtrBarA = 1, kCtrBarD = 2, kCtrBarC = 3, kCtrInts = 8;

constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kBoxes * kQBox;           // 73728
constexpr int kOffP = kOffKV + kBoxes * kKVBox;          // 184320: [hi b0, hi b1, lo b0, lo b1]
constexpr int kOffSel = kOffP + 4 * kPBlk;               // 217088: selected bits
constexpr int kOffTpos = kOffSel + kMaxWords * 4;        // [kTile] positions of the tile rows
constexpr int kOffTrow = kOffTpos + kTile * 4;           // [kTile] cache rows of the tile
constexpr int kOffAlpha = kOffTrow + kTile * 4;          // [64]
constexpr int kOffScan = kOffAlpha + kHB * 4;            // block scan buffer
constexpr int kOffMisc = kOffScan + 128;                 // shared scalars
constexpr int kOffBar = kOffMisc + 128;
constexpr int kNumBars = 6;
constexpr int kOffTmem = kOffBar + 8 * kNumBars;
constexpr int kSmemUsed = kOffTmem + 16;
constexpr int kSmemBytes = kSmemUsed + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
// Phase-B scratch (member list, fallback histogram) and the merge weights
// live in the P region, which phase C writes only after them.
static_assert(kMemberMax * 8 + 160 * 4 <= 4 * kPBlk, "member list and chunk counts fit the P region");
static_assert(2048 * 4 <= 4 * kPBlk, "fallback histogram fits the P region");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // S: 96 columns (M = 64 layout)
constexpr uint32_t kColO = 128;    // O^T blocks at 128, 192, 256, 320
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kHB) | (1u << 15);  // A MN-major

// Shared scalars.
enum {
  kMAbort, kMBin, kMAbove, kMInBin, kMB2, kMAbove2, kMC2, kMNm, kMThKey, kMThPos
};

struct TailParams {
  const int32_t* q_offsets;
  CacheLayout cache;
  const int32_t* ctx_lens;
  const __nv_bfloat16* kv;
  const float* scores;
  long long ld;
  const int* hist;        // [Nq][4096] score-key histograms built by the indexer
  int* fine;              // [Nq][2048] sub-histograms of the threshold bin (zeroed)
  int* ctr;               // [Nq][kCtrInts] counters (zeroed)
  uint32_t* cand_key;     // [Nq][kCandMax]
  int* cand_pos;          // [Nq][kCandMax]
  int* chunk_nsure;       // [Nq][C] sure positions per chunk
  float* part_o;          // [Nq][C][64][512] unnormalised partial outputs
  float2* part_ml;        // [Nq][C][64] (max in log2 units, sum)
  int32_t* idx;
  float* out;
  float* lse;
  unsigned* err;
  int B, Nq, H, top_k, C;
  float scale_log2;
  int select_only;  // stop after writing the index sets (the attention runs separately)
};

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Thread 0 only: arrive on a row counter and wait (bounded) until `target`
// CTAs have arrived.  Returns false if the wait ran out or an error was
// recorded elsewhere.
__device__ bool row_arrive_wait(int* ctr, int target, unsigned* err) {
  __threadfence();
  atomicAdd(ctr, 1);
  const long long t0 = clock64();
  for (unsigned it = 1;; ++it) {
    if (ld_acquire(ctr) >= target) break;
    if ((it & 15u) == 0u) {
      if (*reinterpret_cast<volatile unsigned*>(err) != 0u) return false;
      if (clock64() - t0 > kWaitCycles) {
        atomicOr(err, kErrTimeout);
        return false;
      }
    }
  }
  __threadfence();
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
    decode_tail_kernel(const __grid_constant__ CUtensorMap qmap, const TailParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const bp = smem_raw + (base - raw);
  const uint32_t sQ = base + kOffQ, sKV = base + kOffKV, sP = base + kOffP;
  uint32_t* const sbits = reinterpret_cast<uint32_t*>(bp + kOffSel);
  int* const tpos = reinterpret_cast<int*>(bp + kOffTpos);
  int* const trow = reinterpret_cast<int*>(bp + kOffTrow);
  float* const alpha_s = reinterpret_cast<float*>(bp + kOffAlpha);
  int* const buf = reinterpret_cast<int*>(bp + kOffScan);
  int* const misc = reinterpret_cast<int*>(bp + kOffMisc);
  const uint32_t bars = base + kOffBar;
  const uint32_t b_qfull = bars, b_kvfull = bars + 8u, b_sfull = bars + 16u,
                 b_pfull = bars + 24u, b_odone = bars + 32u, b_drain = bars + 40u;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(bp + kOffTmem);

  const int tid = threadIdx.x;
  const int warp = warp_id_uniform();
  const int lane = lane_id();
  const int r = blockIdx.x / P.C;
  const int c = blockIdx.x - r * P.C;
  const unsigned lt = (1u << lane) - 1u;

  if (tid == 0) {
    mbar_init(b_qfull, 1);
    mbar_init(b_kvfull, kThreads);
    mbar_init(b_sfull, 1);
    mbar_init(b_pfull, kSoftThreads);
    mbar_init(b_odone, 1);
    mbar_init(b_drain, 1);
    fence_mbar_init();
    misc[kMAbort] = 0;
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  // The queries and the batch arrays are inputs of the layer, final before
  // the indexer ran: load and look them up while the indexer finishes.
  if (warp == 4 && lane == 0 && !P.select_only) {
    tma_prefetch_map(&qmap);
    mbar_arrive_expect_tx(b_qfull, kBoxes * kQBox);
    const uint64_t pol = l2_policy_evict_first();
    for (int j = 0; j < kBoxes; ++j) {
      tma_load_2d(sQ + j * kQBox, &qmap, b_qfull, 64 * j, r * P.H, pol);
    }
  }
  const RowSeq rs = row_seq_warp(P.q_offsets, P.cache, P.ctx_lens, P.B, r);
  pdl_wait();
  pdl_launch_dependents();
  if (tid == 0 && error_recorded(P.err)) misc[kMAbort] = 1;

  const int n = rs.len;  // causal length p + 1
  const int k = P.top_k;
  const bool full = n <= k;  // every causal position is kept
  const int S = ((n + P.C - 1) / P.C + 31) & ~31;
  const int s0 = c * S;
  const int s1 = min(n, s0 + S);
  const int nw = s1 > s0 ? (s1 - s0 + 31) >> 5 : 0;  // <= kMaxWords (host condition)
  const float* const sc = P.scores + static_cast<size_t>(r) * P.ld;
  int* const ctr = P.ctr + static_cast<size_t>(r) * kCtrInts;
  int32_t* const idx_row = P.idx + static_cast<size_t>(r) * k;
  __syncthreads();
  bool ok = misc[kMAbort] == 0;

  // ---------------------------------------------------------- phase A ----
  int c_above = 0, c_in = 0;
  uint32_t bstar = 0;
  if (ok && !full) {
    // The first pass's scores (one 32-position word per warp step, kWordsPerWarp
    // per warp) in flight at once, together with the histogram loads below.
    float sv[kWordsPerWarp];
    auto load_pass = [&](int wbase) {
#pragma unroll
      for (int i = 0; i < kWordsPerWarp; ++i) {
        const int w = wbase + warp + i * kWarps;
        const int s = s0 + 32 * w + lane;
        sv[i] = (w < nw && s < s1) ? __ldcg(sc + s) : 0.f;
      }
    };
    load_pass(0);
    // Bin of the k-th largest key: thread t holds bins 8u .. 8u+7 (u = 511 - t),
    // so the exclusive prefix in thread order counts the keys in higher bins.
    const int u = kThreads - 1 - tid;
    const int* const gh = P.hist + static_cast<size_t>(r) * kHistBins;
    const int4 h0 = __ldcg(reinterpret_cast<const int4*>(gh) + 2 * u);
    const int4 h1 = __ldcg(reinterpret_cast<const int4*>(gh) + 2 * u + 1);
    const int cb[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
    int tot = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) tot += cb[j];
    int total;
    int above = block_excl_sum_nw<kWarps>(tot, buf, total);
    if (above < k && k <= above + tot) {
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        if (above + cb[j] >= k) {
          misc[kMBin] = 8 * u + j;
          misc[kMAbove] = above;
          misc[kMInBin] = cb[j];
          break;
        }
        above += cb[j];
      }
    }
    __syncthreads();
    bstar = static_cast<uint32_t>(misc[kMBin]);
    c_above = misc[kMAbove];
    c_in = misc[kMInBin];
    int* const fine = P.fine + static_cast<size_t>(r) * kFineBins;
    uint32_t* const ck = P.cand_key + static_cast<size_t>(r) * kCandMax;
    int* const cp = P.cand_pos + static_cast<size_t>(r) * kCandMax;
    int* const wcnt = reinterpret_cast<int*>(alpha_s);  // [kWarps] counts, then bases
#pragma unroll 1
    for (int wbase = 0; wbase < nw; wbase += kWordsPerWarp * kWarps) {
      if (wbase > 0) load_pass(wbase);
      // Classify: sure and candidate bits per word; the rows of both start
      // coming into L2 now; candidates are counted into the row's
      // sub-histogram (reductions, nothing waits on them).
      int n_cand = 0;
#pragma unroll
      for (int i = 0; i < kWordsPerWarp; ++i) {
        const int w = wbase + warp + i * kWarps;
        if (w >= nw) break;
        const int s = s0 + 32 * w + lane;
        const bool in = s < s1;
        const uint32_t key = score_key(sv[i]);
        const uint32_t bin = key >> kHistShift;
        const bool gt = in && bin > bstar;
        const bool eq = in && bin == bstar;
        const unsigned mg = __ballot_sync(0xffffffffu, gt);
        const unsigned me = __ballot_sync(0xffffffffu, eq);
        if (lane == 0) sbits[w] = mg;
        if (gt || eq) {
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                           P.kv + static_cast<size_t>(seq_row(rs.rows, s)) * kLatent),
                       "r"(kLatent * 2)
                       : "memory");
        }
        if (eq) atomicAdd(fine + ((key >> kFineShift) & (kFineBins - 1)), 1);
        n_cand += __popc(me);
      }
      // One reservation in the row's candidate list per pass for the whole CTA.
      if (lane == 0) wcnt[warp] = n_cand;
      __syncthreads();
      if (tid == 0) {
        int sum = 0;
        for (int w = 0; w < kWarps; ++w) sum += wcnt[w];
        int at = sum > 0 ? atomicAdd(ctr + kCtrCand, sum) : 0;
        for (int w = 0; w < kWarps; ++w) {
          const int cnt = wcnt[w];
          wcnt[w] = at;
          at += cnt;
        }
      }
      __syncthreads();
      int at = wcnt[warp];
#pragma unroll
      for (int i = 0; i < kWordsPerWarp; ++i) {
        const int w = wbase + warp + i * kWarps;
        if (w >= nw) break;
        const int s = s0 + 32 * w + lane;
        const uint32_t key = score_key(sv[i]);
        const bool eq = s < s1 && (key >> kHistShift) == bstar;
        const unsigned me = __ballot_sync(0xffffffffu, eq);
        if (eq) {
          const int slot = at + __popc(me & lt);
          if (slot < kCandMax) {
            ck[slot] = key;
            cp[slot] = s;
          }
        }
        at += __popc(me);
      }
      __syncthreads();  // the counts area is reused by the next pass
    }
  } else if (ok) {
    for (int w = tid; w < nw; w += kThreads) {
      const int rem = s1 - (s0 + 32 * w);
      const uint32_t m = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
      sbits[w] = m;
    }
  }
  __syncthreads();
  // The number of sure positions of the chunk, for the output offsets.
  {
    const uint32_t sw = (ok && !full && tid < nw) ? sbits[tid] : 0u;
    int n_sure;
    block_excl_sum_nw<kWarps>(__popc(sw), buf, n_sure);
    if (tid == 0 && ok && !full) P.chunk_nsure[static_cast<size_t>(r) * P.C + c] = n_sure;
  }
  __syncthreads();

  // Arrive on the row counter as soon as this CTA's phase-A writes (the
  // candidates, the sub-histogram counts, the chunk's count) are issued, and
  // wait for the row's other CTAs.
  bool row_ok = true;
  if (ok && !full && tid == 0) {
    if (!row_arrive_wait(ctr + kCtrBarA, P.C, P.err)) row_ok = false;
  }
  __syncwarp();  // warp 0 meets the CTA barrier reconverged
  ok = ok && !__syncthreads_or(!row_ok);

  // ---------------------------------------------------------- phase B ----
  // own: every chunk of the row holds at most kTile selected positions, and
  // this CTA attends over its own chunk's (n_own of them, in tpos) with no
  // further row barrier.  The decision is the same in every CTA of the row.
  bool own = false;
  int n_own = 0;
  if (ok && !full) {
    const int need = k - c_above;  // keys to keep from the threshold bin, 1 .. c_in
    const bool listed = c_in <= kCandMax;  // every candidate of the row is in the list
    // Everything phase B reads, in flight at once: the sub-histogram, the
    // row's candidates (batches of kCandPer per thread; usually one batch,
    // which then stays in registers for both passes) and the earlier chunks'
    // counts.
    const uint32_t* const ck = P.cand_key + static_cast<size_t>(r) * kCandMax;
    const int* const cp = P.cand_pos + static_cast<size_t>(r) * kCandMax;
    const int n_batches = listed ? (c_in + kCandPer * kThreads - 1) / (kCandPer * kThreads) : 0;
    uint32_t ckr[kCandPer];
    int cpr[kCandPer];
    auto load_batch = [&](int bt) {
#pragma unroll
      for (int i = 0; i < kCandPer; ++i) {
        const int j = (bt * kCandPer + i) * kThreads + tid;
        const bool in = listed && j < c_in;
        ckr[i] = in ? __ldcg(ck + j) : 0u;
        cpr[i] = in ? __ldcg(cp + j) : -1;
      }
    };
    load_batch(0);
    const int nsure_t = tid < P.C ? __ldcg(P.chunk_nsure + static_cast<size_t>(r) * P.C + tid) : 0;
    const int nsure_before = tid < c ? nsure_t : 0;
    int* const ccount = reinterpret_cast<int*>(bp + kOffP + kMemberMax * 8);  // [C]
    // Sub-bin of the need-th key of the bin: thread t holds sub-bins 4u .. 4u+3.
    {
      const int u = kThreads - 1 - tid;
      const int4 f = __ldcg(reinterpret_cast<const int4*>(P.fine + static_cast<size_t>(r) *
                                                                       kFineBins) + u);
      const int tot = f.x + f.y + f.z + f.w;
      int total;
      const int above = block_excl_sum_nw<kWarps>(tot, buf, total);
      if (above < need && need <= above + tot) {
        if (above + f.w >= need) {
          misc[kMB2] = 4 * u + 3; misc[kMAbove2] = above; misc[kMC2] = f.w;
        } else if (above + f.w + f.z >= need) {
          misc[kMB2] = 4 * u + 2; misc[kMAbove2] = above + f.w; misc[kMC2] = f.z;
        } else if (above + f.w + f.z + f.y >= need) {
          misc[kMB2] = 4 * u + 1; misc[kMAbove2] = above + f.w + f.z; misc[kMC2] = f.y;
        } else {
          misc[kMB2] = 4 * u; misc[kMAbove2] = above + f.w + f.z + f.y; misc[kMC2] = f.x;
        }
      }
      if (tid == 0) misc[kMNm] = 0;
      for (int i = tid; i < P.C; i += kThreads) ccount[i] = 0;
      __syncthreads();
    }
    const uint32_t b2 = static_cast<uint32_t>(misc[kMB2]);
    const int need2 = need - misc[kMAbove2];  // members of the sub-bin to keep
    const bool fallback = !listed || misc[kMC2] > kMemberMax;  // the same row-wide
    if (!fallback) {
      uint32_t* const mk = reinterpret_cast<uint32_t*>(bp + kOffP);
      int* const mp = reinterpret_cast<int*>(mk + kMemberMax);
#pragma unroll 1
      for (int bt = 0; bt < n_batches; ++bt) {
        if (bt > 0) load_batch(bt);
#pragma unroll
        for (int i = 0; i < kCandPer; ++i) {
          if (cpr[i] >= 0 && ((ckr[i] >> kFineShift) & (kFineBins - 1)) == b2) {
            const int at = atomicAdd(&misc[kMNm], 1);
            if (at < kMemberMax) {
              mk[at] = ckr[i];
              mp[at] = cpr[i];
            }
          }
        }
      }
      __syncthreads();
      const int nm = min(misc[kMNm], kMemberMax);
      // The need2-th best member (key desc, position asc) is the cut.
      for (int i = tid; i < nm; i += kThreads) {
        int rank = 0;
        for (int j = 0; j < nm; ++j) {
          rank += mk[j] > mk[i] || (mk[j] == mk[i] && mp[j] < mp[i]);
        }
        if (rank == need2 - 1) {
          misc[kMThKey] = static_cast<int>(mk[i]);
          misc[kMThPos] = mp[i];
        }
      }
      __syncthreads();
      const uint32_t th_key = static_cast<uint32_t>(misc[kMThKey]);
      const int th_pos = misc[kMThPos];
      // Selected candidates: this chunk's into the selected bits, earlier
      // chunks' counted for the output offset.
      int before = nsure_before;
#pragma unroll 1
      for (int bt = 0; bt < n_batches; ++bt) {
        if (n_batches > 1) load_batch(bt);
#pragma unroll
        for (int i = 0; i < kCandPer; ++i) {
          const uint32_t key = ckr[i];
          const int pos = cpr[i];
          const uint32_t sub = (key >> kFineShift) & (kFineBins - 1);
          const bool selc =
              pos >= 0 && (sub > b2 || (sub == b2 && (key > th_key ||
                                                       (key == th_key && pos <= th_pos))));
          if (selc) {
            atomicAdd(&ccount[pos / S], 1);
            if (pos < s0) {
              ++before;
            } else if (pos < s1) {
              atomicOr(&sbits[(pos - s0) >> 5], 1u << ((pos - s0) & 31));
            }
          }
        }
      }
      __syncthreads();
      own = !__syncthreads_or(tid < P.C && nsure_t + ccount[tid] > kTile);
      if (tid < kTile) tpos[tid] = -1;
      int offset;
      block_excl_sum_nw<kWarps>(before, buf, offset);
      __syncthreads();
      // This chunk's selected positions, in order, at `offset` (and, when
      // attending over the own chunk, at 0.. in tpos).
      const uint32_t sw = tid < nw ? sbits[tid] : 0u;
      int n_sel_chunk;
      const int lx = block_excl_sum_nw<kWarps>(__popc(sw), buf, n_sel_chunk);
      const int ex = offset + lx;
      uint32_t m = sw;
      for (int j = 0; m != 0u; ++j) {
        const int bit = __ffs(m) - 1;
        m &= m - 1u;
        const int pos = s0 + 32 * tid + bit;
        if (ex + j < k) idx_row[ex + j] = pos;
        if (own) tpos[lx + j] = pos;  // lx + j < n_sel_chunk <= kTile
      }
      n_own = n_sel_chunk;
    } else if (c == 0) {
      // Heavily tied row: the row's first CTA selects over the whole row.
      int* const fh = reinterpret_cast<int*>(bp + kOffP);
      row_select_global<kWarps>(sc, n, k, idx_row, fh, buf);
    }
  } else if (ok && full) {
    // Every position is kept, in its own slot; the padding past n from the
    // first CTA.
    for (int i = s0 + tid; i < s1; i += kThreads) idx_row[i] = i;
    if (c == 0) {
      for (int i = n + tid; i < k; i += kThreads) idx_row[i] = -1;
    }
  }
  __syncthreads();
  // Selection only: the index sets are written; phases C and D are skipped
  // (the rows that phase A started bringing into L2 serve the attention).
  if (P.select_only) ok = false;
  // The row's index set is complete once every CTA of the row has written its
  // part (rows that keep every position need no wait: slot i holds i).
  if (ok && !full && !own && tid == 0) {
    if (!row_arrive_wait(ctr + kCtrBarC, P.C, P.err)) row_ok = false;
  }
  __syncwarp();
  ok = ok && !__syncthreads_or(!row_ok);

  // ---------------------------------------------------------- phase C ----
  // The own chunk's selected positions (one tile), or else this CTA's equal
  // share of the row's selected slots, in tiles of kTile.
  const int n_sel = min(k, n);
  const int share = (n_sel + P.C - 1) / P.C;
  const int slot_lo = min(n_sel, c * share);
  const int slot_hi = min(n_sel, slot_lo + share);
  const int n_tiles = !ok ? 0 : own ? (n_own > 0 ? 1 : 0) : (slot_hi - slot_lo + kTile - 1) / kTile;
  // Positions and cache rows of tile t, -1 past its end.
  auto map_tile = [&](int t) {
    if (tid < kTile) {
      int pos;
      if (own) {
        pos = tpos[tid];
      } else {
        const int g = slot_lo + t * kTile + tid;
        pos = g < slot_hi ? (full ? g : __ldcg(idx_row + g)) : -1;
        tpos[tid] = pos;
      }
      trow[tid] = pos >= 0 ? static_cast<int>(seq_row(rs.rows, pos)) : -1;
    }
  };
  // The tile's rows in 16-byte pieces (cp.async, 128-byte swizzle): thread
  // (sub, piece) copies piece `piece` of every box of rows sub, sub + 64: a
  // warp instruction reads four whole 128-byte lines, its four swizzled rows
  // cover every shared-memory bank four times, and the swizzle (row & 7 ==
  // sub & 7) is fixed per thread.  Every thread arrives on kv_full once its
  // copies have landed.
  // Only the ncol rows the products read are copied (zeros past the tile's
  // own rows).
  auto gather_tile = [&](int ncol) {
    const uint32_t piece = static_cast<uint32_t>(tid & 7);
    const int sub = tid >> 3;
    const uint32_t sw = (piece ^ static_cast<uint32_t>(sub & 7)) << 4;
    for (int i = sub; i < ncol; i += kThreads >> 3) {
      const int row = trow[i];
      const uint32_t dst = sKV + i * 128 + sw;
      if (row >= 0) {
        const __nv_bfloat16* src = P.kv + static_cast<size_t>(row) * kLatent + piece * 8;
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx) cp_async16_tc(dst + bx * kKVBox, src + bx * 64);
      } else {
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx) {
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst + bx * kKVBox), "r"(0u)
                       : "memory");
        }
      }
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    fence_proxy_async_smem();
    mbar_arrive(b_kvfull);
  };
  // Warp 4: S = Q K_tile^T for the gathered tile t (its first ncol rows).
  auto issue_s = [&](int t, int ncol) -> bool {
    bool good = __all_sync(0xffffffffu, mbar_wait(b_qfull, 0, P.err));
    good = good && __all_sync(0xffffffffu, mbar_wait(b_kvfull, static_cast<uint32_t>(t & 1), P.err));
    if (!good) return false;
    tc_fence_after();
    const uint64_t dq = sdesc_sw128(sQ), dk = sdesc_sw128(sKV);
#pragma unroll 4
    for (int ks = 0; ks < kLatent / 16; ++ks) {
      const uint32_t off = (ks & 3) * 32;
      tc_mma_bf16_warp(tmem + kColS, dq + static_cast<uint64_t>(((ks >> 2) * kQBox + off) >> 4),
                       dk + static_cast<uint64_t>(((ks >> 2) * kKVBox + off) >> 4),
                       idesc_bf16_f32(64, static_cast<uint32_t>(ncol)),
                       ks > 0 ? 1u : 0u);
    }
    tc_commit_warp(b_sfull);
    return true;
  };

  float m_run = -INFINITY, l_run = 0.f;
  const int q4 = warp;  // softmax warps 0-3: TMEM lane quadrant
  const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
  const bool owner = lane < 16;
  const int hl = 16 * q4 + (lane & 15);
  for (int t = 0; t < n_tiles && ok; ++t) {
    if (t > 0) {  // the previous tile's products must be done with KV, S and P
      const bool good = mbar_wait(b_odone, static_cast<uint32_t>((t - 1) & 1), P.err);
      ok = !__syncthreads_or(!good);
      if (!ok) break;
      tc_fence_after();
    }
    // Rows of this tile, and the product width: a multiple of 16 covering them.
    const int rows_t = own ? n_own : min(kTile, slot_hi - slot_lo - t * kTile);
    const int ncol = min(kTile, max(16, (rows_t + 15) & ~15));
    map_tile(t);
    __syncthreads();
    gather_tile(ncol);
    if (warp == 4 && !issue_s(t, ncol)) row_ok = false;
    if (warp < 4) {
      // ------------------------------------------------------- softmax --
      const bool good = mbar_wait(b_sfull, static_cast<uint32_t>(t & 1), P.err);
      if (good) {
        tc_fence_after();
        uint32_t va[32], vb[16];
        tmem_ld_16x32bx2_x32<kHalf>(tmem + lane_base + kColS, va);
        tmem_ld_16x32bx2_x16<kHalf>(tmem + lane_base + kColS + 32u, vb);
        tmem_ld_wait();
        const unsigned v0 = __ballot_sync(0xffffffffu, tpos[lane] >= 0);
        const unsigned v1 = __ballot_sync(0xffffffffu, tpos[32 + lane] >= 0);
        const unsigned v2 = __ballot_sync(0xffffffffu, tpos[64 + lane] >= 0);
        const int k0 = (lane >> 4) * kHalf;
        const unsigned long long valid =
            k0 == 0 ? (static_cast<unsigned long long>(v1 & 0xFFFFu) << 32) | v0
                    : (static_cast<unsigned long long>(v2) << 16) | (v1 >> 16);
        float s[kHalf];
        float tmax = -INFINITY;
#pragma unroll
        for (int kk = 0; kk < kHalf; ++kk) {
          const float raw_s = __uint_as_float(kk < 32 ? va[kk] : vb[kk - 32]);
          s[kk] = ((valid >> kk) & 1ull) ? raw_s * P.scale_log2 : -INFINITY;
          tmax = fmaxf(tmax, s[kk]);
        }
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
        const bool raise = tmax > m_run + kRescaleLog2 || (m_run == -INFINITY && tmax > -INFINITY);
        const float m_new = raise ? tmax : m_run;
        const float alpha = (raise && m_run != -INFINITY) ? exp2_fast(m_run - m_new) : 1.f;
        const float m_ref = m_new == -INFINITY ? 0.f : m_new;
        float sum = 0.f;
        uint32_t hi[kHalf / 2], lo[kHalf / 2];
#pragma unroll
        for (int kk = 0; kk < kHalf; kk += 2) {
          const float p0 = exp2_fast(s[kk] - m_ref);
          const float p1 = exp2_fast(s[kk + 1] - m_ref);
          sum += p0 + p1;
          const uint32_t h2 = pack2_bf16(p0, p1);
          hi[kk / 2] = h2;
          lo[kk / 2] = pack2_bf16(p0 - __uint_as_float(h2 << 16),
                                  p1 - __uint_as_float(h2 & 0xFFFF0000u));
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 16);
        l_run = l_run * alpha + sum;
        m_run = m_new;
        if (owner) alpha_s[hl] = alpha;
        // P^T rows (one per head), keys in 16-byte chunks of 8: chunk j of this
        // half is key chunk (k0 / 8 + j), in block (chunk / 8).
#pragma unroll
        for (int j = 0; j < kHalf / 8; ++j) {
          const int ch = k0 / 8 + j;
          const uint32_t blk = static_cast<uint32_t>(ch >> 3);
          const uint32_t off = static_cast<uint32_t>(((ch & 7) ^ (hl & 7)) << 4);
          const uint32_t row_hi = sP + blk * kPBlk + hl * 128;
          const uint32_t row_lo = row_hi + 2 * kPBlk;
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(row_hi + off),
                       "r"(hi[4 * j]), "r"(hi[4 * j + 1]), "r"(hi[4 * j + 2]), "r"(hi[4 * j + 3])
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(row_lo + off),
                       "r"(lo[4 * j]), "r"(lo[4 * j + 1]), "r"(lo[4 * j + 2]), "r"(lo[4 * j + 3])
                       : "memory");
        }
        fence_proxy_async_smem();
      }
      // Rescale O^T (columns = heads) where a head's running max rose.
      const bool any = named_bar_or(1, kSoftThreads, (owner && t > 0 && alpha_s[hl] != 1.f) || !good);
      if (good && any) {
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            uint32_t o[32];
            const uint32_t ta = tmem + lane_base + kColO + 64u * blk + 32u * half;
            tmem_ld_32x32b_x32(ta, o);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha_s[32 * half + j]);
            }
            tmem_st_32x32b_x32(ta, o);
          }
        }
        tmem_st_wait();
      }
      tc_fence_before();
      if (good) mbar_arrive(b_pfull);
      if (!good) row_ok = false;
    } else if (warp == 4) {
      // ---------------------------------------------------------- P.V --
      const bool good = __all_sync(0xffffffffu, mbar_wait(b_pfull, static_cast<uint32_t>(t & 1), P.err));
      if (good) {
        tc_fence_after();
        const uint64_t dv = sdesc_sw128_mn(sKV, kKVBox);
        const uint64_t dp = sdesc_sw128(sP);
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
#pragma unroll 2
          for (int kk = 0; kk < ncol / 16; ++kk) {
            const uint64_t a = dv + static_cast<uint64_t>(((2 * blk) * kKVBox + kk * 2048) >> 4);
            const uint32_t d = tmem + kColO + 64u * blk;
            const uint64_t bo =
                static_cast<uint64_t>(((kk >> 2) * kPBlk + (kk & 3) * 32) >> 4);
            tc_mma_bf16_warp(d, a, dp + bo, kIdescPV, (t > 0 || kk > 0) ? 1u : 0u);
            tc_mma_bf16_warp(d, a, dp + static_cast<uint64_t>((2 * kPBlk) >> 4) + bo, kIdescPV,
                             1u);
          }
        }
        tc_commit_warp(b_odone);
      } else {
        row_ok = false;
      }
    }
    ok = ok && !__syncthreads_or(!row_ok);
  }

  // ---------------------------------------- partial results of the chunk ----
  // Every warp stores a quarter of its TMEM lane quadrant's share: warps w,
  // w+4, w+8, w+12 read quadrant w % 4, two (block, half) pieces each.
  const size_t rec = (static_cast<size_t>(r) * P.C + c) * kHB;
  if (ok) {
    bool good = true;
    if (n_tiles > 0) good = mbar_wait(b_odone, static_cast<uint32_t>((n_tiles - 1) & 1), P.err);
    if (good) {
      tc_fence_after();
      if (n_tiles > 0) {
        const uint32_t qbase = static_cast<uint32_t>((warp & 3) * 32) << 16;
#pragma unroll 1
        for (int piece = 2 * (warp >> 2); piece < 2 * (warp >> 2) + 2; ++piece) {
          const int blk = piece >> 1, half = piece & 1;
          uint32_t o[32];
          tmem_ld_32x32b_x32(tmem + qbase + kColO + 64u * blk + 32u * half, o);
          tmem_ld_wait();
          const int dv = 128 * blk + 32 * (warp & 3) + lane;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int h = 32 * half + j;
            if (h < P.H) __stcg(P.part_o + (rec + h) * kValue + dv, __uint_as_float(o[j]));
          }
        }
      }
      if (warp < 4 && owner && hl < P.H) P.part_ml[rec + hl] = make_float2(m_run, l_run);
    } else {
      row_ok = false;
    }
  }
  ok = ok && !__syncthreads_or(!row_ok);
  if (ok && tid == 0) {
    if (!row_arrive_wait(ctr + kCtrBarD, P.C, P.err)) misc[kMAbort] = 1;
  }
  __syncwarp();
  __syncthreads();
  ok = ok && misc[kMAbort] == 0;

  // ---------------------------------------------------------- phase D ----
  if (ok) {
    const int U = P.H * (kValue / 4);  // float4 units of the row's output
    const int per = (U + P.C - 1) / P.C;
    const int u0 = c * per, u1 = min(U, u0 + per);
    if (u0 < u1) {
      const int hlo = u0 / (kValue / 4), hhi = (u1 - 1) / (kValue / 4);
      float* const wgt = reinterpret_cast<float*>(bp + kOffP);  // [hhi - hlo + 1][C]
      const float2* const ml = P.part_ml + static_cast<size_t>(r) * P.C * kHB;
      for (int h = hlo + warp; h <= hhi; h += kWarps) {
        float M = -INFINITY;
        for (int j = lane; j < P.C; j += 32) M = fmaxf(M, __ldcg(ml + static_cast<size_t>(j) * kHB + h).x);
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o2));
        float L = 0.f;
        for (int j = lane; j < P.C; j += 32) {
          const float2 v = __ldcg(ml + static_cast<size_t>(j) * kHB + h);
          const float wj = v.x == -INFINITY ? 0.f : exp2f(v.x - M);
          wgt[(h - hlo) * P.C + j] = wj;
          L += wj * v.y;
        }
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o2);
        const float inv = L > 0.f ? 1.f / L : 0.f;
        for (int j = lane; j < P.C; j += 32) wgt[(h - hlo) * P.C + j] *= inv;
        if (lane == 0 && P.lse && u0 <= h * (kValue / 4)) {
          P.lse[static_cast<size_t>(r) * P.H + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
        }
      }
      __syncthreads();
      // G threads per output unit (a float4 of one head), each summing every
      // G-th chunk's partial with its loads in flight together, combined with
      // shuffles; chunks in a fixed order, so the result is deterministic.
      // Units beyond kThreads / G per pass take further passes.
      const int nu = u1 - u0;
      int G = 1;
      while (G < 32 && 2 * G * nu <= kThreads) G *= 2;
      const int per_pass = kThreads / G;
      const int sub = tid % G;
#pragma unroll 1
      for (int ub = 0; ub < nu; ub += per_pass) {
        const int ui = ub + tid / G;
        const bool act = ui < nu;
        const int u = u0 + (act ? ui : 0);
        const int h = u / (kValue / 4);
        const int d4 = u - h * (kValue / 4);
        const float* const wr = wgt + (h - hlo) * P.C;
        const float* const po =
            P.part_o + (static_cast<size_t>(r) * P.C * kHB + h) * kValue + 4 * d4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        constexpr int kU = 10;
#pragma unroll 1
        for (int j0 = sub; j0 < P.C; j0 += kU * G) {
          float4 x[kU];
#pragma unroll
          for (int jj = 0; jj < kU; ++jj) {
            const int j = j0 + jj * G;
            x[jj] = (act && j < P.C && wr[j] != 0.f)
                        ? __ldcg(reinterpret_cast<const float4*>(po + static_cast<size_t>(j) *
                                                                          kHB * kValue))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int jj = 0; jj < kU; ++jj) {
            const int j = j0 + jj * G;
            const float wj = (act && j < P.C) ? wr[j] : 0.f;
            acc.x = fmaf(wj, x[jj].x, acc.x);
            acc.y = fmaf(wj, x[jj].y, acc.y);
            acc.z = fmaf(wj, x[jj].z, acc.z);
            acc.w = fmaf(wj, x[jj].w, acc.w);
          }
        }
        for (int o2 = 1; o2 < G; o2 <<= 1) {  // the G threads of a unit are adjacent lanes
          acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o2);
          acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o2);
          acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o2);
          acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o2);
        }
        if (act && sub == 0) {
          *reinterpret_cast<float4*>(P.out + (static_cast<size_t>(r) * P.H + h) * kValue +
                                     4 * d4) = acc;
        }
      }
    }
  }

  // -------------------------------------------------------------- exit ----
  // Nothing this CTA issued (the Q load, the gathers, the MMAs) may still be
  // running when it exits.
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  if (warp == 4) {
    tc_commit_warp(b_drain);
    if (lane == 0) {
      mbar_drain(b_drain, 0, P.err);
      if (!P.select_only) mbar_drain(b_qfull, 0, P.err);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int decode_tail_chunks(int Nq, int num_sms) { return std::max(1, num_sms / std::max(1, Nq)); }

bool decode_tail_fits(int Nq, int64_t max_len, int num_sms) {
  const int C = decode_tail_chunks(Nq, num_sms);
  return Nq > 0 && Nq <= 16 && C >= 8 &&
         ((max_len + C - 1) / C + 31) / 32 <= kMaxWords;
}

bool decode_tail_supported(int Nq, int H, int64_t max_len, int num_sms) {
  const int C = decode_tail_chunks(Nq, num_sms);
  // Measured on B200 (one layer call, L2 flushed): the fused tail is faster
  // than the separate selection, attention and merge kernels for 6 to 12
  // rows; with fewer rows its per-row merge over C = 148 / Nq partials, with
  // more its single tile per chunk, cost more than the extra launches.
  return Nq >= 6 && Nq <= 12 && H <= kHB && C >= 8 &&
         ((max_len + C - 1) / C + 31) / 32 <= kMaxWords;
}

size_t decode_tail_zero_bytes(int Nq) {
  return static_cast<size_t>(Nq) * (kHistBins + kFineBins + kCtrInts) * sizeof(int);
}

size_t decode_tail_ws_bytes(int Nq, int C) {
  return decode_tail_zero_bytes(Nq) +
         static_cast<size_t>(Nq) * kCandMax * (sizeof(uint32_t) + sizeof(int)) +
         static_cast<size_t>(Nq) * C * sizeof(int) +
         static_cast<size_t>(Nq) * C * kHB * (kValue * sizeof(float) + sizeof(float2)) + 256;
}

cudaError_t launch_decode_tail(const DecodeTailArgs& a, cudaStream_t stream) {
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
  cudaError_t e = ensure_smem_limit<decode_tail_kernel>(kSmemBytes);
  if (e == cudaSuccess) e = prefer_max_shared(reinterpret_cast<const void*>(decode_tail_kernel));
  if (e != cudaSuccess) return e;
  const int C = decode_tail_chunks(a.Nq, a.num_sms);
  TailParams P;
  P.q_offsets = a.q_offsets;
  P.cache = a.cache;
  P.ctx_lens = a.ctx_lens;
  P.kv = reinterpret_cast<const __nv_bfloat16*>(a.kv);
  P.scores = a.scores;
  P.ld = a.ld;
  uint8_t* p = static_cast<uint8_t*>(a.ws_region);
  P.hist = reinterpret_cast<const int*>(p);
  p += static_cast<size_t>(a.Nq) * kHistBins * sizeof(int);
  P.fine = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(a.Nq) * kFineBins * sizeof(int);
  P.ctr = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(a.Nq) * kCtrInts * sizeof(int);
  P.cand_key = reinterpret_cast<uint32_t*>(p);
  p += static_cast<size_t>(a.Nq) * kCandMax * sizeof(uint32_t);
  P.cand_pos = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(a.Nq) * kCandMax * sizeof(int);
  P.chunk_nsure = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(a.Nq) * C * sizeof(int);
  p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 255) & ~uintptr_t(255));
  P.part_o = reinterpret_cast<float*>(p);
  p += static_cast<size_t>(a.Nq) * C * kHB * kValue * sizeof(float);
  P.part_ml = reinterpret_cast<float2*>(p);
  P.idx = a.idx;
  P.out = a.out;
  P.lse = a.lse;
  P.err = a.err;
  P.B = a.B;
  P.Nq = a.Nq;
  P.H = a.H;
  P.top_k = a.top_k;
  P.C = C;
  P.scale_log2 = a.scale * kLog2e;
  P.select_only = a.select_only ? 1 : 0;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.Nq * C));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  // The CTAs of a row wait for one another: the launch must make them all
  // resident at once (one CTA per SM, Nq x C <= the SM count).
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, decode_tail_kernel, qmap, P);
}

}  // namespace dsa
