// C ABI of the DSA layer: argument validation, workspace layout and launch
// sequencing.  Every entry point validates everything it is given before it
// enqueues any work, so a failing call leaves all outputs untouched.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <set>
#include <utility>

#include "../../include/dsa.h"
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      return nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

cudaError_t prefer_max_shared(const void* kernel) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({kernel, dev}) != 0) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done.insert({kernel, dev});
  return e;
}

namespace {

// Zeroes `words` 32-bit words at `p` as a programmatic dependent launch: it
// waits for the kernels before it (they may still read the region) and lets
// the next kernel's CTAs start their set-up at once.  A memset node in the
// stream instead makes the next kernel wait for it to finish before its
// launch begins.
__global__ void __launch_bounds__(256) zero_words_kernel(uint32_t* p, size_t words) {
  pdl_wait();
  pdl_launch_dependents();
  const size_t n4 = words / 4;
  uint4* const p4 = reinterpret_cast<uint4*>(p);
  for (size_t i = blockIdx.x * 256 + threadIdx.x; i < n4; i += static_cast<size_t>(gridDim.x) * 256) {
    p4[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  for (size_t i = n4 * 4 + blockIdx.x * 256 + threadIdx.x; i < words;
       i += static_cast<size_t>(gridDim.x) * 256) {
    p[i] = 0u;
  }
}

// `bytes` (a multiple of 4) at the 16-byte aligned `p`.
cudaError_t zero_async(void* p, size_t bytes, cudaStream_t st) {
  if (bytes == 0) return cudaSuccess;
  const size_t words = bytes / 4;
  const unsigned grid = static_cast<unsigned>(std::min<size_t>((words / 4 + 255) / 256 + 1, 148));
  return launch_pdl(zero_words_kernel, dim3(grid), dim3(256), 0, st, 0,
                    static_cast<uint32_t*>(p), words);
}

}  // namespace

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dsa_status check_batch(const dsa_batch* b, BatchInfo* info) {
  if (!b || b->B < 0 || b->Nq < 0) return DSA_ERR_INVALID_ARG;
  info->max_len = 0;
  info->cache_rows = 0;
  info->page_shift = 0;
  if (b->page_size < 0) return DSA_ERR_INVALID_ARG;
  const bool paged = b->page_size > 0;
  if (paged) {
    if (b->page_size < 64 || (b->page_size & (b->page_size - 1)) != 0) return DSA_ERR_UNSUPPORTED;
    while ((1 << info->page_shift) < b->page_size) ++info->page_shift;
  }
  if (b->B == 0) return b->Nq == 0 ? DSA_OK : DSA_ERR_INVALID_ARG;
  if (!b->q_offsets || !b->ctx_lens || !b->h_q_offsets || !b->h_ctx_lens) {
    return DSA_ERR_INVALID_ARG;
  }
  if (b->h_q_offsets[0] != 0 || b->h_q_offsets[b->B] != b->Nq) return DSA_ERR_INVALID_ARG;
  if (paged) {
    if (!b->block_table || !b->h_block_table || b->max_blocks < 1 || b->cache_rows <= 0 ||
        b->cache_rows % b->page_size != 0) {
      return DSA_ERR_INVALID_ARG;
    }
    info->cache_rows = b->cache_rows;
  } else {
    if (!b->kv_offsets || !b->h_kv_offsets || b->h_kv_offsets[0] < 0) return DSA_ERR_INVALID_ARG;
    info->cache_rows = b->h_kv_offsets[b->B];
  }
  const int64_t pages = paged ? b->cache_rows / b->page_size : 0;
  for (int i = 0; i < b->B; ++i) {
    const int64_t nq = static_cast<int64_t>(b->h_q_offsets[i + 1]) - b->h_q_offsets[i];
    const int64_t L = b->h_ctx_lens[i];
    if (nq < 0 || L < 0 || nq > L) return DSA_ERR_INVALID_ARG;
    if (paged) {
      const int64_t used = (L + b->page_size - 1) / b->page_size;
      if (used > b->max_blocks) return DSA_ERR_INVALID_ARG;
      const int32_t* bt = b->h_block_table + static_cast<int64_t>(i) * b->max_blocks;
      for (int64_t j = 0; j < used; ++j) {
        if (bt[j] < 0 || bt[j] >= pages) return DSA_ERR_INVALID_ARG;
      }
    } else {
      const int64_t cap = b->h_kv_offsets[i + 1] - b->h_kv_offsets[i];
      if (cap < 0 || L > cap) return DSA_ERR_INVALID_ARG;
    }
    if (L > info->max_len) info->max_len = L;
  }
  // Row coordinates of the tensor maps are 32-bit.
  if (info->cache_rows >= (int64_t(1) << 31) ||
      static_cast<int64_t>(b->Nq) * kIdxHeads >= (int64_t(1) << 31)) {
    return DSA_ERR_UNSUPPORTED;
  }
  return DSA_OK;
}

dsa_status check_topk(int top_k) {
  if (top_k < 1) return DSA_ERR_INVALID_ARG;
  if (top_k > kMaxTopK) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

dsa_status check_heads(int H) {
  if (H < 1) return DSA_ERR_INVALID_ARG;
  if (H > kMaxHeads) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

dsa_status check_ptr(const void* p) {
  if (!p) return DSA_ERR_INVALID_ARG;
  return aligned16(p) ? DSA_OK : DSA_ERR_UNSUPPORTED;
}

// The current device must be compute capability 10.0 (B200, sm_100a code).
dsa_status check_device(int* num_sms) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return DSA_ERR_NOT_SM100;
  }
  static int cached_sms[64];
  static int cached_ok[64];  // 0 unknown, 1 sm_100, 2 other
  static std::mutex mu;
  if (dev >= 0 && dev < 64) {
    std::lock_guard<std::mutex> lock(mu);
    if (cached_ok[dev] == 0) {
      int major = 0, minor = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return DSA_ERR_CUDA;
      }
      cached_ok[dev] = (major == 10 && minor == 0) ? 1 : 2;
      cached_sms[dev] = sms;
    }
    if (cached_ok[dev] != 1) return DSA_ERR_NOT_SM100;
    *num_sms = cached_sms[dev];
    return DSA_OK;
  }
  return DSA_ERR_NOT_SM100;
}

namespace {

// Split planning uses a fixed SM count so workspace sizes do not depend on
// which device (or whether any device) is present.
constexpr int kPlanSms = 148;

// Workspace: [control 256 B][scores][top-k histograms and candidate lists]
// [attention partials]; the middle regions exist for dsa_layer_forward only.
struct WsLayout {
  size_t scores_off, scores_bytes, hist_off, hist_bytes, part_off, part_bytes, total;
  int64_t ld;
  bool hist_topk;   // selection driven by histograms the indexer builds
  bool fused_tail;  // ... and everything after the indexer in one kernel
  bool select_tail; // ... or the selection in that kernel, the attention after it
  AttnPlan plan;
};

// Few long rows (decode, one or a few new tokens per sequence): the indexer
// builds the score-key histograms and the selection makes one filtering pass.
bool plan_hist_topk(const dsa_batch* b, const BatchInfo& info, int top_k) {
  return b->Nq > 0 && b->Nq <= kPlanSms && info.max_len >= 8192 &&
         info.max_len >= 4LL * top_k &&
         topk_hist_supported(b->Nq, info.max_len);
}

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// dsa_masked_attn: the control block and the chunks' partial results.
size_t masked_ws_need(const dsa_batch* b, const BatchInfo& info, int H) {
  const AttnPlan p = masked_attn_plan(b->Nq, H, info.max_len, kPlanSms);
  return kControlBytes + round_up(attn_partial_bytes(b->Nq, H, p), 256);
}

// Workspace bytes of the standalone calls with DSA_FLAG_SCORE_HISTOGRAM: the
// control block, then the histogram region (the histograms and counters
// first, the selection's lists after them).
size_t standalone_hist_need(const dsa_batch* b, const BatchInfo& info, int top_k) {
  return kControlBytes + round_up(topk_hist_ws_bytes(b->Nq, top_k, info.max_len), 256);
}

WsLayout plan_ws(const dsa_batch* b, const BatchInfo& info, int H, int top_k, bool scores,
                 bool attn) {
  WsLayout w;
  w.ld = static_cast<int64_t>(round_up(static_cast<size_t>(info.max_len), 4));
  w.scores_off = kControlBytes;
  w.scores_bytes = scores ? round_up(static_cast<size_t>(b->Nq) * w.ld * sizeof(float), 256) : 0;
  w.hist_topk = scores && plan_hist_topk(b, info, top_k);
  w.fused_tail = w.hist_topk && attn && decode_tail_supported(b->Nq, H, info.max_len, kPlanSms);
  // The tail's selection alone (then the separate attention) measured faster
  // than the filter and emit kernels for 13 to 16 rows, and no faster for 5
  // or fewer.
  w.select_tail = w.hist_topk && attn && !w.fused_tail && b->Nq > 12 &&
                  decode_tail_fits(b->Nq, info.max_len, kPlanSms);
  w.hist_off = w.scores_off + w.scores_bytes;
  w.hist_bytes =
      (w.fused_tail || w.select_tail)
          ? round_up(decode_tail_ws_bytes(b->Nq, decode_tail_chunks(b->Nq, kPlanSms)), 256)
          : (w.hist_topk ? round_up(topk_hist_ws_bytes(b->Nq, top_k, info.max_len), 256) : 0);
  w.part_off = w.hist_off + w.hist_bytes;
  w.plan = attn_plan(b->Nq, H, top_k, kPlanSms);
  w.part_bytes = attn && !w.fused_tail ? round_up(attn_partial_bytes(b->Nq, H, w.plan), 256) : 0;
  w.total = w.part_off + w.part_bytes;
  // The standalone calls with DSA_FLAG_SCORE_HISTOGRAM keep the histogram
  // region right after the control block.
  if (scores && attn) {
    w.total = std::max(w.total, standalone_hist_need(b, info, top_k));
  }
  return w;
}

dsa_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws || ws_bytes < need) return DSA_ERR_WORKSPACE;
  if (!aligned16(ws)) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

CacheLayout cache_layout(const dsa_batch* b, const BatchInfo& info) {
  CacheLayout c;
  const bool paged = b->page_size > 0;
  c.kv_offsets = paged ? nullptr : b->kv_offsets;
  c.block_table = paged ? b->block_table : nullptr;
  c.max_blocks = paged ? b->max_blocks : 0;
  c.page_shift = info.page_shift;
  return c;
}

inline dsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

inline unsigned* err_word(void* ws) {
  return &reinterpret_cast<Control*>(ws)->err;
}

#define DSA_TRY(expr)                  \
  do {                                 \
    const dsa_status s_ = (expr);      \
    if (s_ != DSA_OK) return s_;       \
  } while (0)

IndexerArgs indexer_args(const dsa_batch* b, const BatchInfo& info, const uint16_t* q_idx,
                         const float* w, const uint16_t* k_idx, float* scores, int64_t ld,
                         void* ws, int num_sms) {
  IndexerArgs a;
  a.B = b->B;
  a.h_q_offsets = b->h_q_offsets;
  a.h_kv_offsets = b->h_kv_offsets;
  a.h_ctx_lens = b->h_ctx_lens;
  a.Nq = b->Nq;
  a.cache_rows = info.cache_rows;
  a.cache = cache_layout(b, info);
  a.q_idx = q_idx;
  a.w = w;
  a.k_idx = k_idx;
  a.scores = scores;
  a.ld = ld;
  a.err = err_word(ws);
  a.num_sms = num_sms;
  a.hist = nullptr;
  a.test_stall = false;
  return a;
}

TopkArgs topk_args(const dsa_batch* b, const BatchInfo& info, const float* scores, int64_t ld,
                   int top_k, int32_t* idx, void* ws, int num_sms) {
  TopkArgs t;
  t.B = b->B;
  t.Nq = b->Nq;
  t.q_offsets = b->q_offsets;
  t.ctx_lens = b->ctx_lens;
  t.scores = scores;
  t.ld = ld;
  t.top_k = top_k;
  t.idx = idx;
  t.max_len = info.max_len;
  t.num_sms = num_sms;
  t.err = err_word(ws);
  return t;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

size_t dsa_workspace_size(const dsa_batch* batch, int H, int top_k, uint32_t flags) {
  BatchInfo info;
  if (check_batch(batch, &info) != DSA_OK || check_heads(H) != DSA_OK ||
      check_topk(top_k) != DSA_OK || (flags & ~DSA_FLAG_MASKED_ROUTE) != 0u) {
    return 0;
  }
  // The layer call and the standalone attention call (whose slice partials
  // the fused layer does not need) on the same workspace.
  size_t total = std::max(plan_ws(batch, info, H, top_k, true, true).total,
                          plan_ws(batch, info, H, top_k, false, true).total);
  if ((flags & DSA_FLAG_MASKED_ROUTE) != 0u) {
    total = std::max(total, masked_ws_need(batch, info, H));
  }
  return total;
}

dsa_status dsa_indexer_score(const dsa_batch* batch, const uint16_t* q_idx, const float* w,
                             const uint16_t* k_idx, float* scores, int64_t ld_scores, void* ws,
                             size_t ws_bytes, uint32_t flags, void* stream) {
  BatchInfo info;
  DSA_TRY(check_batch(batch, &info));
  if ((flags & ~DSA_FLAG_SCORE_HISTOGRAM) != 0u) return DSA_ERR_INVALID_ARG;
  const bool hist = (flags & DSA_FLAG_SCORE_HISTOGRAM) != 0u;
  if (batch->Nq == 0) return DSA_OK;
  DSA_TRY(check_ptr(q_idx));
  DSA_TRY(check_ptr(w));
  DSA_TRY(check_ptr(k_idx));
  DSA_TRY(check_ptr(scores));
  if (ld_scores < info.max_len || (ld_scores & 3) != 0) return DSA_ERR_INVALID_ARG;
  DSA_TRY(check_ws(ws, ws_bytes, hist ? kControlBytes + topk_hist_zero_bytes(batch->Nq)
                                      : kControlBytes));
  int sms = 0;
  DSA_TRY(check_device(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  IndexerArgs ia = indexer_args(batch, info, q_idx, w, k_idx, scores, ld_scores, ws, sms);
  if (hist) {
    void* const region = static_cast<uint8_t*>(ws) + kControlBytes;
    DSA_TRY(cuda_status(zero_async(region, topk_hist_zero_bytes(batch->Nq), st)));
    ia.hist = static_cast<int*>(region);
  }
  return cuda_status(launch_indexer_score(ia, st));
}

dsa_status dsa_topk(const dsa_batch* batch, const float* scores, int64_t ld_scores, int top_k,
                    int32_t* idx, void* ws, size_t ws_bytes, uint32_t flags, void* stream) {
  BatchInfo info;
  DSA_TRY(check_batch(batch, &info));
  DSA_TRY(check_topk(top_k));
  if ((flags & ~DSA_FLAG_SCORE_HISTOGRAM) != 0u) return DSA_ERR_INVALID_ARG;
  if (batch->Nq == 0) return DSA_OK;
  DSA_TRY(check_ptr(scores));
  DSA_TRY(check_ptr(idx));
  if (ld_scores < info.max_len || (ld_scores & 3) != 0) return DSA_ERR_INVALID_ARG;
  // The histogram path where the fused layer would take it, given the flag.
  const bool hist = (flags & DSA_FLAG_SCORE_HISTOGRAM) != 0u &&
                    plan_hist_topk(batch, info, top_k);
  DSA_TRY(check_ws(ws, ws_bytes,
                   hist ? standalone_hist_need(batch, info, top_k) : kControlBytes));
  int sms = 0;
  DSA_TRY(check_device(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const TopkArgs a = topk_args(batch, info, scores, ld_scores, top_k, idx, ws, sms);
  if (!hist) return cuda_status(launch_topk(a, st));
  // The filter accumulates into the sub-histograms and counters that follow
  // the histograms: clear those, so the same histograms serve every call.
  uint8_t* const region = static_cast<uint8_t*>(ws) + kControlBytes;
  const size_t hist_bytes = static_cast<size_t>(batch->Nq) * kHistBins * sizeof(int);
  DSA_TRY(cuda_status(zero_async(region + hist_bytes,
                                 topk_hist_zero_bytes(batch->Nq) - hist_bytes, st)));
  return cuda_status(launch_topk_hist(a, region, st));
}

dsa_status dsa_sparse_attn(const dsa_batch* batch, const uint16_t* q, int H, const uint16_t* kv,
                           const int32_t* idx, int top_k, float scale, float* out, float* lse,
                           void* ws, size_t ws_bytes, void* stream) {
  BatchInfo info;
  DSA_TRY(check_batch(batch, &info));
  DSA_TRY(check_heads(H));
  DSA_TRY(check_topk(top_k));
  if (batch->Nq == 0) return DSA_OK;
  DSA_TRY(check_ptr(q));
  DSA_TRY(check_ptr(kv));
  DSA_TRY(check_ptr(idx));
  DSA_TRY(check_ptr(out));
  if (lse) DSA_TRY(check_ptr(lse));
  if (!isfinite(scale)) return DSA_ERR_INVALID_ARG;
  const WsLayout L = plan_ws(batch, info, H, top_k, false, true);
  DSA_TRY(check_ws(ws, ws_bytes, L.total));
  int sms = 0;
  DSA_TRY(check_device(&sms));
  AttnArgs a;
  a.B = batch->B;
  a.Nq = batch->Nq;
  a.q_offsets = batch->q_offsets;
  a.cache = cache_layout(batch, info);
  a.q = q;
  a.H = H;
  a.kv = kv;
  a.idx = idx;
  a.top_k = top_k;
  a.scale = scale;
  a.out = out;
  a.lse = lse;
  a.part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.part_off);
  a.err = err_word(ws);
  a.ctx_lens = batch->ctx_lens;
  a.idx_prefix = false;
  a.batch_ready = false;
  a.cache_rows = info.cache_rows;
  a.plan = L.plan;
  return cuda_status(launch_sparse_attn(a, static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_masked_attn(const dsa_batch* batch, const uint16_t* q, int H, const uint16_t* kv,
                           const int32_t* idx, int top_k, float scale, float* out, float* lse,
                           void* ws, size_t ws_bytes, void* stream) {
  BatchInfo info;
  DSA_TRY(check_batch(batch, &info));
  DSA_TRY(check_heads(H));
  DSA_TRY(check_topk(top_k));
  if (batch->Nq == 0) return DSA_OK;
  DSA_TRY(check_ptr(q));
  DSA_TRY(check_ptr(kv));
  DSA_TRY(check_ptr(idx));
  DSA_TRY(check_ptr(out));
  if (lse) DSA_TRY(check_ptr(lse));
  if (!isfinite(scale)) return DSA_ERR_INVALID_ARG;
  // Contiguous caches only: the route streams each sequence's rows as tiles.
  if (!masked_attn_supported(info.max_len) || batch->page_size > 0) return DSA_ERR_UNSUPPORTED;
  DSA_TRY(check_ws(ws, ws_bytes, masked_ws_need(batch, info, H)));
  int sms = 0;
  DSA_TRY(check_device(&sms));
  AttnArgs a;
  a.B = batch->B;
  a.Nq = batch->Nq;
  a.q_offsets = batch->q_offsets;
  a.cache = cache_layout(batch, info);
  a.ctx_lens = batch->ctx_lens;
  a.q = q;
  a.H = H;
  a.kv = kv;
  a.idx = idx;
  a.top_k = top_k;
  a.scale = scale;
  a.out = out;
  a.lse = lse;
  a.part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kControlBytes);
  a.err = err_word(ws);
  a.idx_prefix = false;
  a.batch_ready = false;
  a.cache_rows = info.cache_rows;
  a.plan = masked_attn_plan(batch->Nq, H, info.max_len, kPlanSms);
  return cuda_status(launch_masked_attn(a, static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_layer_forward(const dsa_batch* batch, const uint16_t* q, int H,
                             const uint16_t* q_idx, const float* w, const uint16_t* k_idx,
                             const uint16_t* kv, int top_k, float scale, float* out, float* lse,
                             int32_t* idx, void* ws, size_t ws_bytes, uint32_t flags,
                             void* stream) {
  BatchInfo info;
  if ((flags & ~DSA_FLAG_TEST_STALL) != 0u) return DSA_ERR_INVALID_ARG;
  DSA_TRY(check_batch(batch, &info));
  DSA_TRY(check_heads(H));
  DSA_TRY(check_topk(top_k));
  if (batch->Nq == 0) return DSA_OK;
  DSA_TRY(check_ptr(q));
  DSA_TRY(check_ptr(q_idx));
  DSA_TRY(check_ptr(w));
  DSA_TRY(check_ptr(k_idx));
  DSA_TRY(check_ptr(kv));
  DSA_TRY(check_ptr(out));
  DSA_TRY(check_ptr(idx));
  if (lse) DSA_TRY(check_ptr(lse));
  if (!isfinite(scale)) return DSA_ERR_INVALID_ARG;
  const WsLayout L = plan_ws(batch, info, H, top_k, true, true);
  DSA_TRY(check_ws(ws, ws_bytes, L.total));
  int sms = 0;
  DSA_TRY(check_device(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* const scores = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.scores_off);

  IndexerArgs ia = indexer_args(batch, info, q_idx, w, k_idx, scores, L.ld, ws, sms);
  ia.test_stall = (flags & DSA_FLAG_TEST_STALL) != 0u;
  void* const hist_region = static_cast<uint8_t*>(ws) + L.hist_off;
  if (L.hist_topk) {
    // The histograms and counters start from zero on every call: no state is
    // carried in the workspace from one call to the next.
    DSA_TRY(cuda_status(zero_async(hist_region,
                                   (L.fused_tail || L.select_tail)
                                       ? decode_tail_zero_bytes(batch->Nq)
                                       : topk_hist_zero_bytes(batch->Nq),
                                   st)));
    ia.hist = static_cast<int*>(hist_region);
  }
  DSA_TRY(cuda_status(launch_indexer_score(ia, st)));
  if (L.fused_tail || L.select_tail) {
    DecodeTailArgs d;
    d.B = batch->B;
    d.Nq = batch->Nq;
    d.H = H;
    d.top_k = top_k;
    d.q_offsets = batch->q_offsets;
    d.cache = cache_layout(batch, info);
    d.ctx_lens = batch->ctx_lens;
    d.q = q;
    d.kv = kv;
    d.scores = scores;
    d.ld = L.ld;
    d.ws_region = hist_region;
    d.idx = idx;
    d.out = out;
    d.lse = lse;
    d.err = err_word(ws);
    d.scale = scale;
    d.num_sms = std::min(sms, kPlanSms);  // the workspace holds kPlanSms / Nq chunks
    d.select_only = L.select_tail;
    DSA_TRY(cuda_status(launch_decode_tail(d, st)));
    if (L.fused_tail) return DSA_OK;
  } else {
    const TopkArgs t = topk_args(batch, info, scores, L.ld, top_k, idx, ws, sms);
    DSA_TRY(
        cuda_status(L.hist_topk ? launch_topk_hist(t, hist_region, st) : launch_topk(t, st)));
  }

  AttnArgs a;
  a.B = batch->B;
  a.Nq = batch->Nq;
  a.q_offsets = batch->q_offsets;
  a.cache = cache_layout(batch, info);
  a.q = q;
  a.H = H;
  a.kv = kv;
  a.idx = idx;
  a.top_k = top_k;
  a.scale = scale;
  a.out = out;
  a.lse = lse;
  a.part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.part_off);
  a.err = err_word(ws);
  a.ctx_lens = batch->ctx_lens;
  a.idx_prefix = true;  // produced by dsa_topk: valid positions first, then -1
  a.batch_ready = true;  // the layer's own kernels never write the batch arrays
  a.cache_rows = info.cache_rows;
  a.plan = L.plan;
  return cuda_status(launch_sparse_attn(a, st));
}

namespace {
inline bool projection_width_ok(int64_t d) { return d >= 64 && d <= 65536 && d % 64 == 0; }
}  // namespace

size_t dsa_indexer_project_workspace_size(const dsa_batch* batch, int64_t d_model, int64_t d_q) {
  BatchInfo info;
  if (check_batch(batch, &info) != DSA_OK || !projection_width_ok(d_model) ||
      !projection_width_ok(d_q)) {
    return 0;
  }
  return kControlBytes + project_ws_bytes(batch->Nq, static_cast<int>(d_q),
                                          static_cast<int>(d_model), kPlanSms);
}

dsa_status dsa_indexer_project(const dsa_batch* batch, const uint16_t* x, int64_t d_model,
                               const uint16_t* c_q, int64_t d_q, const uint16_t* w_q_b,
                               const uint16_t* w_k, const uint16_t* w_proj, uint16_t* q_idx,
                               uint16_t* k_idx, float* w, void* ws, size_t ws_bytes,
                               void* stream) {
  BatchInfo info;
  DSA_TRY(check_batch(batch, &info));
  if (!projection_width_ok(d_model) || !projection_width_ok(d_q)) return DSA_ERR_UNSUPPORTED;
  if (batch->Nq == 0) return DSA_OK;
  const void* ptrs[] = {x, c_q, w_q_b, w_k, w_proj, q_idx, k_idx, w};
  for (const void* p : ptrs) DSA_TRY(check_ptr(p));
  // Split planning uses kPlanSms, so the workspace size does not depend on the device.
  const size_t need = kControlBytes + project_ws_bytes(batch->Nq, static_cast<int>(d_q),
                                                       static_cast<int>(d_model), kPlanSms);
  DSA_TRY(check_ws(ws, ws_bytes, need));
  int sms = 0;
  DSA_TRY(check_device(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProjectArgs a;
  a.B = batch->B;
  a.T = batch->Nq;
  a.q_offsets = batch->q_offsets;
  a.cache = cache_layout(batch, info);
  a.ctx_lens = batch->ctx_lens;
  a.x = x;
  a.c_q = c_q;
  a.w_q_b = w_q_b;
  a.w_k = w_k;
  a.w_proj = w_proj;
  a.d_model = static_cast<int>(d_model);
  a.d_q = static_cast<int>(d_q);
  a.q_idx = q_idx;
  a.k_cache = k_idx;
  a.w = w;
  a.ws_region = static_cast<uint8_t*>(ws) + kControlBytes;
  a.err = err_word(ws);
  a.num_sms = kPlanSms;
  // The split-K tickets start from zero on every call.
  DSA_TRY(cuda_status(zero_async(a.ws_region,
                                 project_zero_bytes(a.T, a.d_q, a.d_model, kPlanSms), st)));
  return cuda_status(launch_indexer_project(a, st));
}

dsa_status dsa_check_device_status(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < kControlBytes) return DSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned host_err = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess ||
      cudaMemcpy(&host_err, err_word(ws), sizeof(host_err), cudaMemcpyDeviceToHost) !=
          cudaSuccess) {
    return DSA_ERR_CUDA;
  }
  if (host_err != 0) {
    if (cudaMemset(err_word(ws), 0, sizeof(unsigned)) != cudaSuccess) return DSA_ERR_CUDA;
    return (host_err & kErrTimeout) != 0u ? DSA_ERR_DEVICE_TIMEOUT : DSA_ERR_BAD_INDEX;
  }
  return DSA_OK;
}

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_DEVICE_TIMEOUT: return "DSA_ERR_DEVICE_TIMEOUT";
    case DSA_ERR_NOT_SM100: return "DSA_ERR_NOT_SM100";
    case DSA_ERR_BAD_INDEX: return "DSA_ERR_BAD_INDEX";
  }
  return "DSA_ERR_UNKNOWN";
}

}  // extern "C"
