// The indexer's input step on tcgen05 tensor cores: for every new token t
//
//   q_idx[t] = c_q[t] . W_q_b^T     (32 x 128 outputs, bf16)
//   k        = x[t]   . W_k^T       (128 outputs, bf16) -> indexer key cache row of t
//   w[t]     = x[t]   . W_proj^T    (32 outputs, fp32)
//
// (llama.cpp b12180 news: aiunderstanding.org "What happened" -- the
// indexer's q_b, k and projection tensors are kept out of quantization;
// devotd.net sections 2-3 -- a DSA layer keeps an indexer key cache.  The
// pages give no widths for x and c_q and no normalisation; the maps are
// taken as plain linear maps.)
//
// The three maps are one GEMM over a concatenated output-feature space of 34
// tiles of 128 features (32 tiles of q_idx, one of k, one of w whose rows past
// 32 are the TMA box's zero fill):
//   D[128 features, N tokens] = W_tile[128, K] . In[N tokens, K]^T
// with the features as M, so a decode step's few tokens still fill the MMA
// (N >= 16) and the weights stream at full width.  Work items are (feature
// tile, token tile, K-slice); with few tokens the K range is split over
// several items so every SM streams weights, each slice's fp32 partial goes
// to the workspace, and the last slice to finish (a per-tile ticket; nobody
// waits) sums the slices in order and runs the epilogue.  The epilogue rounds
// to bf16 and writes k straight into the key cache at the token's row: the
// append is part of the step.
//
// CTA roles (192 threads, one CTA per SM, persistent): warp 0 TMA producer
// (weight tile 16 KB + input tile through a kStages ring, 128-byte swizzle),
// warp 1 TMEM allocation and MMA issue (double-buffered accumulator), warps
// 2-5 epilogue (one TMEM lane -- one feature -- per thread).
#include <string.h>

#include <algorithm>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kFeatTiles = (kIdxHeads * kIdxDim + kIdxDim + 128) / 128;  // 34
constexpr int kTileQ = kIdxHeads * kIdxDim / 128;                        // 32 q_idx tiles
constexpr int kKStep = 64;                 // K per stage (one 128-byte swizzle box)
constexpr int kABytes = 128 * kKStep * 2;  // 16 KB weight tile
constexpr int kStages = 4;
constexpr int kEpiThreads = 128;
constexpr int kThreads = 64 + kEpiThreads;
constexpr int kMaxN = 128;                 // tokens per item

struct ProjParams {
  const int32_t* q_offsets;
  CacheLayout cache;
  const int32_t* ctx_lens;
  int B, T;                  // sequences, tokens (query rows)
  int N;                     // tokens per item (16..128, multiple of 16)
  int n_ttiles;              // token tiles
  int ksplit_q, ksplit_x;    // K slices per q_idx tile / per k, w tile
  int kq_steps, kx_steps;    // 64-wide K steps of c_q and of x
  int n_items;
  uint16_t* q_idx;           // [T][4096]
  uint16_t* k_cache;         // [rows][128]
  float* w;                  // [T][32]
  float* part;               // split partials [tile][token tile][slice][128][N]
  int* tickets;              // [tile][token tile], zeroed
  unsigned* err;
};

struct Item {
  int ft, tt, slice, nslice, k0, k1;  // feature tile, token tile, K slice, K steps [k0, k1)
};

__device__ __forceinline__ Item decode_proj_item(const ProjParams& P, int item) {
  // Items: every (tile, token tile) of the q_idx tiles first, then k and w.
  Item it;
  const int nq_items = kTileQ * P.n_ttiles * P.ksplit_q;
  int rem;
  if (item < nq_items) {
    it.nslice = P.ksplit_q;
    it.ft = item / (P.n_ttiles * P.ksplit_q);
    rem = item - it.ft * P.n_ttiles * P.ksplit_q;
  } else {
    const int j = item - nq_items;
    it.nslice = P.ksplit_x;
    it.ft = kTileQ + j / (P.n_ttiles * P.ksplit_x);
    rem = j - (it.ft - kTileQ) * P.n_ttiles * P.ksplit_x;
  }
  it.tt = rem / it.nslice;
  it.slice = rem - it.tt * it.nslice;
  const int steps = it.ft < kTileQ ? P.kq_steps : P.kx_steps;
  const int per = (steps + it.nslice - 1) / it.nslice;
  it.k0 = it.slice * per;
  it.k1 = min(steps, it.k0 + per);
  return it;
}

__device__ __forceinline__ void named_bar_sync_p(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Cache row of token (query row) t: the row of its position in its sequence.
__device__ __forceinline__ long long token_cache_row(const ProjParams& P, int t) {
  int lo = 0, hi = P.B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(P.q_offsets + mid) <= t) lo = mid; else hi = mid - 1;
  }
  const int q0 = __ldg(P.q_offsets + lo), q1 = __ldg(P.q_offsets + lo + 1);
  const SeqRows sr =
      seq_rows(P.cache, lo, P.cache.block_table ? 0 : __ldg(P.cache.kv_offsets + lo));
  return seq_row(sr, __ldg(P.ctx_lens + lo) - (q1 - q0) + (t - q0));
}

template <int N>
struct ProjCfg {
  static constexpr int kBBytes = N * kKStep * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kSmemData = kStages * kStageBytes;
  static constexpr int kBarBytes = 8 * (2 * kStages + 5) + 16;
  static constexpr int kSmemBytes = kSmemData + kBarBytes + 1024;
  static constexpr int kTmemCols = 2 * N < 32 ? 32 : 2 * N;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(128, N);
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
    indexer_project_kernel(const __grid_constant__ CUtensorMap map_wq,
                           const __grid_constant__ CUtensorMap map_wk,
                           const __grid_constant__ CUtensorMap map_wp,
                           const __grid_constant__ CUtensorMap map_cq,
                           const __grid_constant__ CUtensorMap map_x,
                           const __grid_constant__ ProjParams P) {
  using C = ProjCfg<N>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const uint32_t bars = base + C::kSmemData;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (kStages + s); };
  auto tfull = [&](int i) { return bars + 8u * (2 * kStages + i); };
  auto tempty = [&](int i) { return bars + 8u * (2 * kStages + 2 + i); };
  const uint32_t drain = bars + 8u * (2 * kStages + 4);
  uint32_t* const tmem_slot =
      reinterpret_cast<uint32_t*>(base_ptr + C::kSmemData + 8 * (2 * kStages + 5));
  __shared__ int s_abort, s_last;

  const int warp = warp_id_uniform();
  const int lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull(i), 1);
      mbar_init(tempty(i), kEpiThreads);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&map_wq);
    tma_prefetch_map(&map_wk);
    tma_prefetch_map(&map_wp);
    tma_prefetch_map(&map_cq);
    tma_prefetch_map(&map_x);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0) s_abort = error_recorded(P.err);
  __syncthreads();
  const bool abort = s_abort != 0;
  const int G = static_cast<int>(gridDim.x);

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0 && !abort) {
      const uint64_t pol_w = l2_policy_evict_first();  // weights are read once per step
      const uint64_t pol_in = l2_policy_evict_last();  // inputs are read by every feature tile
      int stage = 0;
      uint32_t sph = 0;
      uint32_t last[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) last[s] = 2u;
      bool ok = true;
      for (int item = blockIdx.x; item < P.n_items && ok; item += G) {
        const Item it = decode_proj_item(P, item);
        const CUtensorMap* wmap =
            it.ft < kTileQ ? &map_wq : (it.ft == kTileQ ? &map_wk : &map_wp);
        const CUtensorMap* imap = it.ft < kTileQ ? &map_cq : &map_x;
        const int wrow = it.ft < kTileQ ? it.ft * 128 : 0;
        for (int ks = it.k0; ks < it.k1; ++ks) {
          ok = mbar_wait(empty(stage), sph ^ 1u, P.err);
          if (!ok) break;
          mbar_arrive_expect_tx(full(stage), C::kStageBytes);
#pragma unroll
          for (int s = 0; s < kStages; ++s) {
            if (s == stage) last[s] = sph;
          }
          const uint32_t dst = base + stage * C::kStageBytes;
          tma_load_2d(dst, wmap, full(stage), ks * kKStep, wrow, pol_w);
          tma_load_2d(dst + kABytes, imap, full(stage), ks * kKStep, it.tt * N, pol_in);
          if (++stage == kStages) {
            stage = 0;
            sph ^= 1u;
          }
        }
      }
#pragma unroll
      for (int s = 0; s < kStages; ++s) {
        if (last[s] != 2u) mbar_drain(full(s), last[s], P.err);
      }
    }
    __syncwarp();  // the warp meets the CTA barrier below reconverged
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0 && !abort) {
      int stage = 0, acc = 0;
      uint32_t sph = 0, aph = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < P.n_items && ok; item += G) {
        const Item it = decode_proj_item(P, item);
        ok = mbar_wait(tempty(acc), aph ^ 1u, P.err);
        if (!ok) break;
        const uint32_t d = tmem + static_cast<uint32_t>(acc * N);
        for (int ks = it.k0; ks < it.k1; ++ks) {
          ok = mbar_wait(full(stage), sph, P.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a = base + stage * C::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < kKStep / 16; ++kk) {
            tc_mma_bf16(d, sdesc_sw128(a + kk * 32), sdesc_sw128(a + kABytes + kk * 32), C::kIdesc,
                        (ks > it.k0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(empty(stage));
          if (++stage == kStages) {
            stage = 0;
            sph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull(acc));
        acc ^= 1;
        if (acc == 0) aph ^= 1u;
      }
      tc_commit(drain);
      mbar_drain(drain, 0, P.err);
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------- epilogue --
    const int quad = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int f_local = quad * 32 + lane;  // this thread's feature within the tile
    int acc = 0;
    uint32_t aph = 0;
    bool ok = !abort;
    for (int item = blockIdx.x; item < P.n_items && ok; item += G) {
      const Item it = decode_proj_item(P, item);
      ok = mbar_wait(tfull(acc), aph, P.err);
      if (!ok) break;
      tc_fence_after();
      const size_t tile = static_cast<size_t>(it.ft) * P.n_ttiles + it.tt;
      // Writes columns c0 .. c0+15 (tokens) of this thread's feature.
      auto emit16 = [&](int c0, const float (&v)[16]) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = it.tt * N + c0 + j;
          if (t < P.T) {
            if (it.ft < kTileQ) {
              P.q_idx[static_cast<size_t>(t) * (kIdxHeads * kIdxDim) + it.ft * 128 + f_local] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
            } else if (it.ft == kTileQ) {
              P.k_cache[token_cache_row(P, t) * kIdxDim + f_local] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
            } else if (f_local < kIdxHeads) {
              P.w[static_cast<size_t>(t) * kIdxHeads + f_local] = v[j];
            }
          }
        }
      };
      auto part_at = [&](int sl, int c0) {
        return P.part + ((tile * it.nslice + sl) * 128 + f_local) * static_cast<size_t>(N) + c0;
      };
#pragma unroll 1
      for (int c0 = 0; c0 < N; c0 += 16) {
        uint32_t r16[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
            "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
            : "=r"(r16[0]), "=r"(r16[1]), "=r"(r16[2]), "=r"(r16[3]), "=r"(r16[4]),
              "=r"(r16[5]), "=r"(r16[6]), "=r"(r16[7]), "=r"(r16[8]), "=r"(r16[9]),
              "=r"(r16[10]), "=r"(r16[11]), "=r"(r16[12]), "=r"(r16[13]), "=r"(r16[14]),
              "=r"(r16[15])
            : "r"(tmem + lane_base + static_cast<uint32_t>(acc * N + c0)));
        tmem_ld_wait();
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r16[j]);
        if (it.nslice == 1) {
          emit16(c0, v);
        } else {  // this slice's partial, for the tile's last slice to sum
          float* const dst = part_at(it.slice, c0);
#pragma unroll
          for (int j = 0; j < 16; j += 4) {
            __stcg(reinterpret_cast<float4*>(dst + j), make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty(acc));
      acc ^= 1;
      if (acc == 0) aph ^= 1u;
      if (it.nslice > 1) {
        // The last slice of the tile to finish (a ticket; nobody waits) sums
        // every slice's partial in slice order and writes the outputs.
        __threadfence();
        named_bar_sync_p(1, kEpiThreads);
        if (threadIdx.x == 64) {
          s_last = atomicAdd(P.tickets + tile, 1) == it.nslice - 1;
          __threadfence();
        }
        named_bar_sync_p(1, kEpiThreads);
        if (s_last != 0) {
#pragma unroll 1
          for (int c0 = 0; c0 < N; c0 += 16) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.f;
            // Eight slices' loads in flight at a time, added in slice order.
            constexpr int kBatch = 8;
#pragma unroll 1
            for (int sl0 = 0; sl0 < it.nslice; sl0 += kBatch) {
              float4 x[kBatch][4];
#pragma unroll
              for (int a = 0; a < kBatch; ++a) {
                const bool in = sl0 + a < it.nslice;
                const float* src = part_at(in ? sl0 + a : 0, c0);
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                  x[a][b] = in ? __ldcg(reinterpret_cast<const float4*>(src + 4 * b))
                               : make_float4(0.f, 0.f, 0.f, 0.f);
                }
              }
#pragma unroll
              for (int a = 0; a < kBatch; ++a) {
                if (sl0 + a < it.nslice) {
#pragma unroll
                  for (int b = 0; b < 4; ++b) {
                    v[4 * b] += x[a][b].x;
                    v[4 * b + 1] += x[a][b].y;
                    v[4 * b + 2] += x[a][b].z;
                    v[4 * b + 3] += x[a][b].w;
                  }
                }
              }
            }
            emit16(c0, v);
          }
        }
        named_bar_sync_p(1, kEpiThreads);  // s_last is read before the next item's ticket
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

inline size_t round_up_256(size_t x) { return (x + 255) / 256 * 256; }

bool encode_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
               uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int N>
cudaError_t launch_n(const ProjectArgs& a, ProjParams P, cudaStream_t stream) {
  using C = ProjCfg<N>;
  CUtensorMap m_wq, m_wk, m_wp, m_cq, m_x;
  if (!encode_2d(&m_wq, a.w_q_b, static_cast<uint64_t>(a.d_q), kIdxHeads * kIdxDim, kKStep, 128) ||
      !encode_2d(&m_wk, a.w_k, static_cast<uint64_t>(a.d_model), kIdxDim, kKStep, 128) ||
      !encode_2d(&m_wp, a.w_proj, static_cast<uint64_t>(a.d_model), kIdxHeads, kKStep, 128) ||
      !encode_2d(&m_cq, a.c_q, static_cast<uint64_t>(a.d_q), static_cast<uint64_t>(a.T), kKStep,
                 N) ||
      !encode_2d(&m_x, a.x, static_cast<uint64_t>(a.d_model), static_cast<uint64_t>(a.T), kKStep,
                 N)) {
    return cudaErrorInvalidValue;
  }
  cudaError_t e = ensure_smem_limit<indexer_project_kernel<N>>(C::kSmemBytes);
  if (e != cudaSuccess) return e;
  P.N = N;
  const int grid = std::min(P.n_items, a.num_sms);
  return launch_pdl(indexer_project_kernel<N>, dim3(grid), dim3(kThreads), C::kSmemBytes, stream,
                    0, m_wq, m_wk, m_wp, m_cq, m_x, P);
}

// Token-tile width and K split of a launch.
void plan_project(int T, int d_q, int d_model, int num_sms, int* N, int* ksq, int* ksx) {
  int n = 16;
  while (n < kMaxN && n < T) n *= 2;
  *N = n;
  const int ttiles = (T + n - 1) / n;
  const int kq = d_q / kKStep, kx = d_model / kKStep;
  *ksq = 1;
  *ksx = 1;
  if ((kTileQ + 2) * ttiles >= num_sms) return;  // whole K ranges already fill the GPU
  // Few tokens: split the K ranges so that the items fit one wave of the SMs
  // and the longest slice (the weight bytes one SM streams) is as short as
  // possible; among equal longest slices, fewer slices (a shorter sum).
  int best = 1 << 30, best_items = 1 << 30;
  for (int q = 1; q <= kq; ++q) {
    const int left = num_sms / ttiles - kTileQ * q;
    if (left < 2) break;
    const int x = std::min(kx, left / 2);
    const int qs = (kq + q - 1) / q;
    int xs = (kx + x - 1) / x;
    int xx = x;
    while (xx > 1 && (kx + xx - 2) / (xx - 1) <= std::max(qs, xs)) {  // no longer a longer slice
      --xx;
    }
    xs = (kx + xx - 1) / xx;
    const int cost = std::max(qs, xs);
    const int items = kTileQ * q + 2 * xx;
    if (cost < best || (cost == best && items < best_items)) {
      best = cost;
      best_items = items;
      *ksq = q;
      *ksx = xx;
    }
  }
}

}  // namespace

size_t project_ws_bytes(int T, int d_q, int d_model, int num_sms) {
  int N, ksq, ksx;
  plan_project(T, d_q, d_model, num_sms, &N, &ksq, &ksx);
  const size_t ttiles = static_cast<size_t>((T + N - 1) / N);
  const size_t tickets = round_up_256(kFeatTiles * ttiles * sizeof(int));
  const size_t parts = (ksq > 1 || ksx > 1)
                           ? static_cast<size_t>(kFeatTiles) * ttiles * std::max(ksq, ksx) * 128 * N *
                                 sizeof(float)
                           : 0;
  return tickets + parts;
}

size_t project_zero_bytes(int T, int d_q, int d_model, int num_sms) {
  int N, ksq, ksx;
  plan_project(T, d_q, d_model, num_sms, &N, &ksq, &ksx);
  const size_t ttiles = static_cast<size_t>((T + N - 1) / N);
  return round_up_256(kFeatTiles * ttiles * sizeof(int));
}

cudaError_t launch_indexer_project(const ProjectArgs& a, cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  int N, ksq, ksx;
  plan_project(a.T, a.d_q, a.d_model, a.num_sms, &N, &ksq, &ksx);
  ProjParams P;
  memset(&P, 0, sizeof(P));
  P.q_offsets = a.q_offsets;
  P.cache = a.cache;
  P.ctx_lens = a.ctx_lens;
  P.B = a.B;
  P.T = a.T;
  P.n_ttiles = (a.T + N - 1) / N;
  P.ksplit_q = ksq;
  P.ksplit_x = ksx;
  P.kq_steps = a.d_q / kKStep;
  P.kx_steps = a.d_model / kKStep;
  P.n_items = (kTileQ * ksq + 2 * ksx) * P.n_ttiles;
  P.q_idx = a.q_idx;
  P.k_cache = a.k_cache;
  P.w = a.w;
  uint8_t* p = static_cast<uint8_t*>(a.ws_region);
  P.tickets = reinterpret_cast<int*>(p);
  P.part = reinterpret_cast<float*>(p + project_zero_bytes(a.T, a.d_q, a.d_model, a.num_sms));
  P.err = a.err;
  switch (N) {
    case 16: return launch_n<16>(a, P, stream);
    case 32: return launch_n<32>(a, P, stream);
    case 64: return launch_n<64>(a, P, stream);
    default: return launch_n<128>(a, P, stream);
  }
}

}  // namespace dsa
