// Lightning-indexer scores on tcgen05 tensor cores.
//
//   I[q, s] = sum_h w[q, h] * ReLU( q_idx[q, h, :] . k_idx[s, :] ),  s <= p(q)
//
// (llama.cpp b12180 news: aiaulis.com paragraph 2 — a light indexer scores
// earlier tokens; devotd.net configuration table — 32 heads, key length 128;
// aiunderstanding.org "What happened" — no RoPE.  The weighted-ReLU form is
// the usual lightning-indexer form, assumed because the pages print none.)
//
// One MMA computes D[128 keys, 32*QT] = K_tile[128 keys, 128] * Q[32*QT, 128]^T
// where the N dimension holds (query, head) pairs of QT queries of one
// sequence.  Keys are the M dimension so that, in the epilogue, each thread
// owns one key (one TMEM lane) and reduces its heads in registers.
//
// CTA roles (192 threads, one CTA per SM, persistent over work items):
//   warp 0     TMA producer: Q block per item, 32 KB K tiles through a
//              kStages-deep ring (128-byte swizzle, two 64-dim boxes).
//   warp 1     TMEM allocation; one thread issues the MMAs (8 x K=16 per
//              tile) into a double-buffered fp32 accumulator in TMEM.
//   warps 2-5  epilogue: tcgen05.ld, ReLU, weighted head sum, fp32 store.
// A work item is (sequence, group of QT queries, chunk of key tiles); items
// are dealt to CTAs in snake order so causal prefill work balances.
//
// Optionally, the epilogue also counts each stored score into its row's
// 4096-bin histogram of the top 12 bits of its order-preserving key; the
// top-k selection then needs only one filtering pass over the row.  With one
// query per item the counts gather in shared memory (one atomic per key) and
// are flushed to the row's histogram after each item; with several queries
// per item (multi-token decode) each warp adds its counts, aggregated per
// distinct bin, to the rows' global histograms directly.
#include <string.h>

#include <algorithm>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kKeysPerTile = 128;
constexpr int kKTileBytes = kKeysPerTile * kIdxDim * 2;  // 32 KB
constexpr int kKBoxBytes = kKTileBytes / 2;              // 128 rows x 64 dims
constexpr int kEpiThreads = 128;  // one epilogue set: a warp per TMEM lane quadrant

struct SeqItems {
  long long kv_off;   // contiguous caches: the sequence's first row
  int q_off, nq, L, n_chunks, item_off, b;
};
static_assert(sizeof(SeqItems) == 32, "packed launch record");

struct IdxParams {
  SeqItems seq[kMaxSeqPerLaunch];
  int nseq, n_items, chunk_tiles, pad;
  const float* w;
  float* scores;
  long long ld;
  unsigned* err;
  int* hist;  // [Nq][kHistBins] score-key histograms, or null
  int stall;  // test only: the TMA producer issues nothing, so every wait runs out
  CacheLayout cache;     // paged caches: the block table (contiguous: kv_off above)
  long long cache_rows;  // rows of k_idx (a row past them reads as zeros)
};

template <int QT>
struct Cfg {
  static constexpr int N = 32 * QT;
  // Epilogue sets: with 4 or 8 queries per item the read-out of a tile takes
  // longer than its MMAs, so two or four sets of four warps split the queries.
  // With one query per item two sets take alternate tiles (set s reads
  // accumulator s), so the read-out, score store and histogram count of a
  // tile overlap the next one's.
  static constexpr bool kSplitTiles = QT == 1;
  static constexpr int kEpiSets = QT >= 8 ? 4 : (QT >= 4 ? 2 : (kSplitTiles ? 2 : 1));
  static constexpr int kThreads = 64 + kEpiSets * kEpiThreads;
  static constexpr int kQBufs = QT <= 4 ? 2 : 1;
  // K ring depth: deep for decode (HBM streaming), shallower when Q is large.
  static constexpr int kStages = QT == 1 ? 5 : (QT == 2 ? 6 : 4);
  static constexpr int kHistBytes = QT == 1 ? kHistBins * 4 : 0;
  static constexpr int kQBoxBytes = N * 128;
  static constexpr int kQBytes = 2 * kQBoxBytes;
  static constexpr int kTmemCols = 2 * N < 32 ? 32 : 2 * N;
  static constexpr int kSmemData = kQBufs * kQBytes + kStages * kKTileBytes + kHistBytes;
  static constexpr int kBarBytes = 8 * (2 * kStages + 9) + 16;
  static constexpr int kSmemBytes = kSmemData + kBarBytes + 1024;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(128, N);
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

struct ItemView {
  int row0, nrow, pos0, kt0, kt1, b;
  long long kv0;
};

template <int QT>
__device__ __forceinline__ bool decode_item(const IdxParams& P, int item, ItemView& v) {
  int b = 0;
  while (b + 1 < P.nseq && P.seq[b + 1].item_off <= item) ++b;
  const SeqItems& s = P.seq[b];
  const int rem = item - s.item_off;
  const int g = rem / s.n_chunks;
  const int c = rem - g * s.n_chunks;
  const int j0 = g * QT;
  v.nrow = min(QT, s.nq - j0);
  v.row0 = s.q_off + j0;
  v.pos0 = s.L - s.nq + j0;
  const int n_kt = (v.pos0 + v.nrow + kKeysPerTile - 1) / kKeysPerTile;
  v.kt0 = c * P.chunk_tiles;
  v.kt1 = min(v.kt0 + P.chunk_tiles, n_kt);
  v.kv0 = s.kv_off;
  v.b = s.b;
  return v.kt0 < v.kt1;
}

__device__ __forceinline__ void named_bar_sync_idx(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Named barrier over `threads` threads; true if `pred` held in any of them.
__device__ __forceinline__ bool named_bar_any(int id, int threads, bool pred) {
  uint32_t res;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(res)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(threads)
      : "memory");
  return res != 0u;
}

__device__ __forceinline__ int snake_item(int j) {
  const int G = static_cast<int>(gridDim.x);
  const int k = static_cast<int>(blockIdx.x);
  return j * G + ((j & 1) ? (G - 1 - k) : k);
}

template <int QT>
__global__ void __launch_bounds__(Cfg<QT>::kThreads, 1)
    indexer_score_kernel(const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap qmap,
                         const __grid_constant__ IdxParams P) {
  using C = Cfg<QT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const uint32_t q_smem = base;
  const uint32_t k_smem = base + C::kQBufs * C::kQBytes;
  int* const shist =
      reinterpret_cast<int*>(base_ptr + C::kQBufs * C::kQBytes + C::kStages * kKTileBytes);
  const uint32_t bars = base + C::kSmemData;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (C::kStages + s); };
  auto qfull = [&](int i) { return bars + 8u * (2 * C::kStages + i); };
  auto qempty = [&](int i) { return bars + 8u * (2 * C::kStages + 2 + i); };
  auto tfull = [&](int i) { return bars + 8u * (2 * C::kStages + 4 + i); };
  auto tempty = [&](int i) { return bars + 8u * (2 * C::kStages + 6 + i); };
  const uint32_t drain = bars + 8u * (2 * C::kStages + 8);  // the MMAs' completion at exit
  uint32_t* const tmem_slot =
      reinterpret_cast<uint32_t*>(base_ptr + C::kSmemData + 8 * (2 * C::kStages + 9));
  __shared__ int s_abort;

  const int warp = warp_id_uniform();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(qfull(i), 1);
      mbar_init(qempty(i), 1);
      mbar_init(tfull(i), 1);
      mbar_init(tempty(i), C::kSplitTiles ? kEpiThreads : C::kEpiSets * kEpiThreads);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&kmap);
    tma_prefetch_map(&qmap);
    // The key tiles of this CTA's first item start coming into L2 while the
    // kernel before this one finishes (a prefetch reads the current data and
    // writes nothing, so it is safe before the dependent-launch wait).
    ItemView v0;
    const int item0 = snake_item(0);
    if (!P.stall && P.cache.block_table == nullptr && item0 < P.n_items &&
        decode_item<QT>(P, item0, v0)) {
      for (int kt = v0.kt0; kt < min(v0.kt1, v0.kt0 + C::kStages + 2); ++kt) {
        const int row = static_cast<int>(v0.kv0 + static_cast<long long>(kt) * kKeysPerTile);
        tma_prefetch_2d(&kmap, 0, row);
        tma_prefetch_2d(&kmap, 64, row);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  // Everything above overlapped the previous kernel; from here on memory is shared.
  pdl_wait();
  pdl_launch_dependents();
  // An error recorded by an earlier kernel: skip the work (every role alike).
  if (threadIdx.x == 0) s_abort = error_recorded(P.err);
  __syncthreads();
  const bool abort = s_abort != 0;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0 && !abort && !P.stall) {
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      int stage = 0, qb = 0;
      uint32_t sph = 0, qph = 0;
      // Parity of the last load issued into each K stage and Q buffer (2: none).
      uint32_t k_last[C::kStages], q_last[2] = {2u, 2u};
#pragma unroll
      for (int st = 0; st < C::kStages; ++st) k_last[st] = 2u;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        const int item = snake_item(j);
        if (item >= P.n_items) break;
        ItemView v;
        if (!decode_item<QT>(P, item, v)) continue;
        ok = mbar_wait(qempty(qb), qph ^ 1u, P.err);
        if (!ok) break;
        mbar_arrive_expect_tx(qfull(qb), C::kQBytes);
        q_last[qb] = qph;
        const uint32_t qdst = q_smem + qb * C::kQBytes;
        tma_load_2d(qdst, &qmap, qfull(qb), 0, v.row0 * kIdxHeads, pol_keep);
        tma_load_2d(qdst + C::kQBoxBytes, &qmap, qfull(qb), 64, v.row0 * kIdxHeads, pol_keep);
        if (++qb == C::kQBufs) {
          qb = 0;
          qph ^= 1u;
        }
        for (int kt = v.kt0; kt < v.kt1; ++kt) {
          ok = mbar_wait(empty(stage), sph ^ 1u, P.err);
          if (!ok) break;
          mbar_arrive_expect_tx(full(stage), kKTileBytes);
#pragma unroll
          for (int st = 0; st < C::kStages; ++st) {
            if (st == stage) k_last[st] = sph;
          }
          const uint32_t kdst = k_smem + stage * kKTileBytes;
          if (P.cache.block_table == nullptr) {
            const int row = static_cast<int>(v.kv0 + static_cast<long long>(kt) * kKeysPerTile);
            tma_load_2d(kdst, &kmap, full(stage), 0, row, pol_stream);
            tma_load_2d(kdst + kKBoxBytes, &kmap, full(stage), 64, row, pol_stream);
          } else {
            // Paged caches: two runs of 64 keys, each inside one page (pages
            // are 64 rows or more); a run past the item's keys reads zeros.
            const int32_t* bt = P.cache.block_table + static_cast<size_t>(v.b) * P.cache.max_blocks;
            const int shift = P.cache.page_shift;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int s = kt * kKeysPerTile + 64 * h;
              const int row = s < v.pos0 + v.nrow
                                  ? (__ldg(bt + (s >> shift)) << shift) + (s & ((1 << shift) - 1))
                                  : static_cast<int>(P.cache_rows);
              tma_load_2d(kdst + h * 64 * 128, &kmap, full(stage), 0, row, pol_stream);
              tma_load_2d(kdst + kKBoxBytes + h * 64 * 128, &kmap, full(stage), 64, row,
                          pol_stream);
            }
          }
          if (++stage == C::kStages) {
            stage = 0;
            sph ^= 1u;
          }
        }
      }
      // Every load issued has landed before the CTA may exit (immediate
      // unless the loops were abandoned).
#pragma unroll
      for (int st = 0; st < C::kStages; ++st) {
        if (k_last[st] != 2u) mbar_drain(full(st), k_last[st], P.err);
      }
      for (int i = 0; i < 2; ++i) {
        if (q_last[i] != 2u) mbar_drain(qfull(i), q_last[i], P.err);
      }
    }
    __syncwarp();  // the warp meets the CTA barrier below reconverged
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0 && !abort) {
      int stage = 0, qb = 0, acc = 0;
      uint32_t sph = 0, qph = 0, aph = 0;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        const int item = snake_item(j);
        if (item >= P.n_items) break;
        ItemView v;
        if (!decode_item<QT>(P, item, v)) continue;
        ok = mbar_wait(qfull(qb), qph, P.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qsrc = q_smem + qb * C::kQBytes;
        for (int kt = v.kt0; kt < v.kt1; ++kt) {
          ok = mbar_wait(tempty(acc), aph ^ 1u, P.err);
          if (!ok) break;
          ok = mbar_wait(full(stage), sph, P.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t ksrc = k_smem + stage * kKTileBytes;
          const uint32_t d = tmem + static_cast<uint32_t>(acc * C::N);
#pragma unroll
          for (int ks = 0; ks < kIdxDim / 16; ++ks) {
            const uint32_t koff = (ks >> 2) * kKBoxBytes + (ks & 3) * 32;
            const uint32_t qoff = (ks >> 2) * C::kQBoxBytes + (ks & 3) * 32;
            tc_mma_bf16(d, sdesc_sw128(ksrc + koff), sdesc_sw128(qsrc + qoff), C::kIdesc,
                        ks > 0 ? 1u : 0u);
          }
          tc_commit(empty(stage));
          tc_commit(tfull(acc));
          if (++stage == C::kStages) {
            stage = 0;
            sph ^= 1u;
          }
          acc ^= 1;
          if (acc == 0) aph ^= 1u;
        }
        if (!ok) break;
        tc_commit(qempty(qb));
        if (++qb == C::kQBufs) {
          qb = 0;
          qph ^= 1u;
        }
      }
      // Every MMA issued has completed before TMEM and the stages are released.
      tc_commit(drain);
      mbar_drain(drain, 0, P.err);
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------- epilogue --
    const int quad = warp & 3;  // TMEM lanes this warp may read: 32*quad ..
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int et = static_cast<int>(threadIdx.x) - 64;  // 0.. over all epilogue sets
    const int jset = (warp - 2) >> 2;                    // this warp's epilogue set
    constexpr int kAllEpi = C::kEpiSets * kEpiThreads;
    const bool do_hist = (QT == 1) && P.hist != nullptr;     // shared-memory histogram
    const bool do_ghist = (QT > 1) && P.hist != nullptr;     // straight to the row's
    if (do_hist) {
      for (int i = et; i < kHistBins; i += kAllEpi) shist[i] = 0;
      named_bar_sync_idx(1, kAllEpi);
    }
    int acc = 0;
    uint32_t aph = 0;
    bool ok = !abort;
    for (int j = 0; ok; ++j) {
      const int item = snake_item(j);
      if (item >= P.n_items) break;
      ItemView v;
      if (!decode_item<QT>(P, item, v)) continue;
      for (int kt = v.kt0; kt < v.kt1; ++kt) {
        if (C::kSplitTiles && acc != jset) {  // the other set's tile
          acc ^= 1;
          if (acc == 0) aph ^= 1u;
          continue;
        }
        ok = mbar_wait(tfull(acc), aph, P.err);
        if (!ok) break;
        tc_fence_after();
        const int key = kt * kKeysPerTile + quad * 32 + lane;
#pragma unroll 1
        for (int jq = C::kSplitTiles ? 0 : jset; jq < QT; jq += C::kSplitTiles ? 1 : C::kEpiSets) {
          if (jq >= v.nrow) break;
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + lane_base + static_cast<uint32_t>(acc * C::N + jq * 32), r);
          tmem_ld_wait();
          const float4* wp =
              reinterpret_cast<const float4*>(P.w + static_cast<size_t>(v.row0 + jq) * kIdxHeads);
          // Four partial sums (heads h = j mod 4), updated two at a time by
          // paired fp32 FMAs: each lane rounds as fmaf does, in the same order.
          float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
          for (int h4 = 0; h4 < kIdxHeads / 4; ++h4) {
            const float4 ww = __ldg(wp + h4);
            ffma2(s0, s1, ww.x, ww.y, fmaxf(__uint_as_float(r[4 * h4 + 0]), 0.f),
                  fmaxf(__uint_as_float(r[4 * h4 + 1]), 0.f));
            ffma2(s2, s3, ww.z, ww.w, fmaxf(__uint_as_float(r[4 * h4 + 2]), 0.f),
                  fmaxf(__uint_as_float(r[4 * h4 + 3]), 0.f));
          }
          float s = (s0 + s1) + (s2 + s3);
          if (s == 0.f) s = 0.f;  // one zero: -0 and +0 are the same score
          const bool valid = key <= v.pos0 + jq;
          if (valid) P.scores[static_cast<size_t>(v.row0 + jq) * P.ld + key] = s;
          if (do_hist) {
            // One shared-memory atomic per key: the keys of a warp are spread
            // over many bins, so they rarely collide.
            if (valid) atomicAdd(&shist[score_key(s) >> kHistShift], 1);
          } else if (do_ghist) {
            // Global atomics are costly: one per distinct bin of the warp.
            const uint32_t bin = valid ? (score_key(s) >> kHistShift) : 0xFFFFFFFFu;
            const unsigned grp = __match_any_sync(0xffffffffu, bin);
            if (valid && lane == __ffs(grp) - 1) {
              atomicAdd(P.hist + static_cast<size_t>(v.row0 + jq) * kHistBins + bin, __popc(grp));
            }
          }
        }
        tc_fence_before();
        mbar_arrive(tempty(acc));
        acc ^= 1;
        if (acc == 0) aph ^= 1u;
      }
      if (do_hist) {  // flush this item's counts into the row's histogram
        // Every set has counted its tiles of the item; a wait that ran out
        // in either set ends both (they meet at every barrier below).
        ok = !named_bar_any(1, kAllEpi, !ok);
        if (ok) {
          int* const gh = P.hist + static_cast<size_t>(v.row0) * kHistBins;
          for (int i = et; i < kHistBins; i += kAllEpi) {
            const int c = shist[i];
            if (c != 0) {
              atomicAdd(gh + i, c);
              shist[i] = 0;
            }
          }
        }
        named_bar_sync_idx(1, kAllEpi);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

bool encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                    uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int QT>
cudaError_t launch_qt(const IndexerArgs& a, cudaStream_t stream) {
  using C = Cfg<QT>;
  CUtensorMap kmap, qmap;
  const bool paged = a.cache.block_table != nullptr;
  if (!encode_bf16_2d(&kmap, a.k_idx, kIdxDim, static_cast<uint64_t>(a.cache_rows), 64,
                      paged ? 64 : kKeysPerTile) ||
      !encode_bf16_2d(&qmap, a.q_idx, kIdxDim, static_cast<uint64_t>(a.Nq) * kIdxHeads, 64,
                      C::N)) {
    return cudaErrorInvalidValue;
  }
  cudaError_t e = ensure_smem_limit<indexer_score_kernel<QT>>(C::kSmemBytes);
  if (e != cudaSuccess) return e;

  // Total key tiles, to size chunks so every SM gets several items.
  long long total_tiles = 0;
  for (int b = 0; b < a.B; ++b) {
    const int nq = a.h_q_offsets[b + 1] - a.h_q_offsets[b];
    const int L = a.h_ctx_lens[b];
    for (int j0 = 0; j0 < nq; j0 += QT) {
      const int nrow = std::min(QT, nq - j0);
      total_tiles += (L - nq + j0 + nrow + kKeysPerTile - 1) / kKeysPerTile;
    }
  }
  const long long target_items = 4LL * a.num_sms;
  // At least 4 tiles per item so a Q reload is amortised over several K tiles.
  const int chunk = static_cast<int>(std::max<long long>(
      4, (total_tiles + target_items - 1) / target_items));

  // Sequences with queries, in launches of at most kMaxSeqPerLaunch.
  int b = 0;
  while (b < a.B) {
    IdxParams P;
    memset(&P, 0, sizeof(P));
    P.chunk_tiles = chunk;
    P.w = a.w;
    P.scores = a.scores;
    P.ld = a.ld;
    P.err = a.err;
    P.hist = a.hist;
    P.stall = a.test_stall ? 1 : 0;
    P.cache = a.cache;
    P.cache_rows = a.cache_rows;
    int items = 0, n = 0;
    for (; b < a.B && n < kMaxSeqPerLaunch; ++b) {
      const int nq = a.h_q_offsets[b + 1] - a.h_q_offsets[b];
      if (nq <= 0) continue;
      SeqItems& r = P.seq[n++];
      r.kv_off = paged ? 0 : a.h_kv_offsets[b];
      r.b = b;
      r.q_off = a.h_q_offsets[b];
      r.nq = nq;
      r.L = a.h_ctx_lens[b];
      const int groups = (nq + QT - 1) / QT;
      const int n_kt_max = (r.L + kKeysPerTile - 1) / kKeysPerTile;
      r.n_chunks = std::max(1, (n_kt_max + chunk - 1) / chunk);
      r.item_off = items;
      items += groups * r.n_chunks;
    }
    P.nseq = n;
    P.n_items = items;
    if (items == 0) continue;
    const int grid = std::min(items, a.num_sms);
    e = launch_pdl(indexer_score_kernel<QT>, dim3(grid), dim3(C::kThreads), C::kSmemBytes, stream, 0,
                   kmap, qmap, P);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_indexer_score(const IndexerArgs& a, cudaStream_t stream) {
  int max_nq = 0;
  for (int b = 0; b < a.B; ++b) max_nq = std::max(max_nq, a.h_q_offsets[b + 1] - a.h_q_offsets[b]);
  if (max_nq <= 1) return launch_qt<1>(a, stream);
  if (max_nq <= 2) return launch_qt<2>(a, stream);
  if (max_nq <= 4) return launch_qt<4>(a, stream);
  return launch_qt<8>(a, stream);
}

}  // namespace dsa
