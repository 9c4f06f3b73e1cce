// Host-side interfaces between the C ABI layer (dsa_api.cu) and the kernel
// translation units.  Arguments here are already validated.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "../../include/dsa.h"

namespace dsa {

// ------------------------------------------------ argument validation ----
// Shared by every entry point; each returns DSA_OK or the status to report.
struct BatchInfo {
  int64_t max_len;     // longest context
  int64_t cache_rows;  // rows of the caches: kv_offsets[B], or the paged caches' rows
  int page_shift;      // log2(page_size) for paged caches, 0 for contiguous ones
};

bool aligned16(const void* p);
// The batch layout (host mirrors) is consistent and within the 32-bit row
// coordinates of the tensor maps; fills `info`.
dsa_status check_batch(const dsa_batch* b, BatchInfo* info);
dsa_status check_topk(int top_k);
dsa_status check_heads(int H);
// Non-null and 16-byte aligned.
dsa_status check_ptr(const void* p);
// The current device is compute capability 10.0; its SM count (cached per
// device) goes to `num_sms`.
dsa_status check_device(int* num_sms);

struct IndexerArgs {
  int B;
  const int32_t* h_q_offsets;   // host mirrors of the batch
  const int64_t* h_kv_offsets;  // contiguous caches (planning only)
  const int32_t* h_ctx_lens;
  int Nq;
  int64_t cache_rows;   // rows of k_idx
  CacheLayout cache;    // device: where each sequence's positions live
  const uint16_t* q_idx;
  const float* w;
  const uint16_t* k_idx;
  float* scores;
  int64_t ld;
  unsigned* err;
  int num_sms;
  int* hist;          // per-row score-key histograms to accumulate, or null
  bool test_stall;    // test only: the TMA producer issues nothing (every wait runs out)
};
cudaError_t launch_indexer_score(const IndexerArgs& a, cudaStream_t stream);

struct TopkArgs {
  int B;
  int Nq;
  const int32_t* q_offsets;   // device
  const int32_t* ctx_lens;    // device
  const float* scores;
  int64_t ld;
  int top_k;
  int32_t* idx;
  int64_t max_len;   // longest context in the batch
  int num_sms;
  unsigned* err;     // workspace error word: the kernels skip their work when it is set
};
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream);
// Selection driven by the histograms the indexer built (see IndexerArgs.hist):
// `ws_region` holds them, the per-row counters and the candidate lists,
// topk_hist_ws_bytes() bytes in all; its first topk_hist_zero_bytes() bytes
// (histograms and counters) must be zero when the indexer starts.
size_t topk_hist_zero_bytes(int Nq);
size_t topk_hist_ws_bytes(int Nq, int top_k, int64_t max_len);
int topk_hist_chunks(int Nq, int64_t max_len, int* chunk_len);
bool topk_hist_supported(int Nq, int64_t max_len);
cudaError_t launch_topk_hist(const TopkArgs& a, void* ws_region, cudaStream_t stream);

// The decode layer after the indexer as one cooperative kernel (selection
// from the indexer's histograms, attention, merge): few long rows with one
// query per sequence and at most 64 heads.
struct DecodeTailArgs {
  int B, Nq, H, top_k;
  const int32_t* q_offsets;   // device
  CacheLayout cache;          // device: where each sequence's positions live
  const int32_t* ctx_lens;    // device
  const uint16_t* q;
  const uint16_t* kv;
  const float* scores;
  int64_t ld;
  void* ws_region;   // decode_tail_ws_bytes; its first decode_tail_zero_bytes zeroed
                     // before the indexer builds the histograms at its start
  int32_t* idx;
  float* out;
  float* lse;
  unsigned* err;
  float scale;
  int num_sms;       // SMs the launch may fill (one CTA per SM)
  bool select_only;  // write the index sets only (q, kv, out, lse unused)
};
int decode_tail_chunks(int Nq, int num_sms);
// The kernel's limits (rows, chunks, chunk length), for either mode.
bool decode_tail_fits(int Nq, int64_t max_len, int num_sms);
// Where the whole fused tail is the faster route.
bool decode_tail_supported(int Nq, int H, int64_t max_len, int num_sms);
size_t decode_tail_zero_bytes(int Nq);
size_t decode_tail_ws_bytes(int Nq, int C);
cudaError_t launch_decode_tail(const DecodeTailArgs& a, cudaStream_t stream);

// The indexer's input step (projections of the new tokens, k appended to the
// indexer key cache) as one tcgen05 GEMM over the concatenated features.
struct ProjectArgs {
  int B, T;                   // sequences, new tokens (query rows)
  const int32_t* q_offsets;   // device
  CacheLayout cache;          // device: where each sequence's positions live
  const int32_t* ctx_lens;    // device
  const uint16_t* x;          // [T][d_model]
  const uint16_t* c_q;        // [T][d_q]
  const uint16_t* w_q_b;      // [4096][d_q]
  const uint16_t* w_k;        // [128][d_model]
  const uint16_t* w_proj;     // [32][d_model]
  int d_model, d_q;           // multiples of 64
  uint16_t* q_idx;            // [T][4096]
  uint16_t* k_cache;          // [rows][128]
  float* w;                   // [T][32]
  void* ws_region;            // project_ws_bytes; its first project_zero_bytes zeroed
  unsigned* err;
  int num_sms;
};
size_t project_ws_bytes(int T, int d_q, int d_model, int num_sms);
size_t project_zero_bytes(int T, int d_q, int d_model, int num_sms);
cudaError_t launch_indexer_project(const ProjectArgs& a, cudaStream_t stream);

// How the attention launch covers (query row, head block, slice of the set).
struct AttnPlan {
  int decode;       // 1: single-tile tcgen05 kernel, slices of 64 slots (few rows)
  int tc;           // 1: tcgen05 kernel (many rows, 64 heads per CTA, no slices)
  int hb;           // heads per CTA: 16, 32, 48 or 64
  int head_blocks;  // ceil(H / hb)
  int n_split;      // slices of the selected set per (row, head block)
  int split_len;    // index slots per slice (multiple of 32)
};
// Plan of the tcgen05 kernel (dsa_sparse_attn, dsa_layer_forward).
AttnPlan attn_plan(int Nq, int H, int top_k, int num_sms);
// Plan of the CUDA-core kernels (16 heads per CTA, slices for few rows).
AttnPlan attn_plan_core(int Nq, int H, int top_k, int num_sms);
size_t attn_partial_bytes(int Nq, int H, const AttnPlan& p);

struct AttnArgs {
  int B;
  int Nq;
  const int32_t* q_offsets;   // device
  CacheLayout cache;          // device: where each sequence's positions live
  const int32_t* ctx_lens;    // device
  const uint16_t* q;
  int H;
  const uint16_t* kv;
  const int32_t* idx;
  int top_k;
  float scale;
  float* out;
  float* lse;
  float* part;        // split partials (workspace); unused when plan.n_split == 1
  unsigned* err;      // workspace error word (bounded waits)
  bool idx_prefix;    // valid entries are the first min(top_k, p+1) slots of each row
  bool batch_ready;   // no kernel this launch depends on writes the batch arrays
  int64_t cache_rows; // rows of kv (the masked route's tensor map)
  AttnPlan plan;
};
cudaError_t launch_sparse_attn_tc(const AttnArgs& a, cudaStream_t stream);
cudaError_t launch_sparse_attn_decode(const AttnArgs& a, cudaStream_t stream);
int attn_decode_slots();  // selected slots per CTA of the single-tile kernel
// Merges the slices of a split launch (plan.n_split > 1) into out and lse.
cudaError_t launch_attn_merge(const AttnArgs& a, cudaStream_t stream);
cudaError_t launch_sparse_attn(const AttnArgs& a, cudaStream_t stream);
// The mask-over-the-whole-cache route (comparison): chunks of the causal
// positions per CTA, every cached row streamed, unlisted rows masked.
AttnPlan masked_attn_plan(int Nq, int H, int64_t max_len, int num_sms);
bool masked_attn_supported(int64_t max_len);
cudaError_t launch_masked_attn(const AttnArgs& a, cudaStream_t stream);

// Raises a kernel's dynamic shared-memory limit to `bytes`, once per device
// (the attribute call is not free, and launches may be captured in a graph).
template <auto Kernel>
cudaError_t ensure_smem_limit(int bytes) {
  static std::atomic<unsigned long long> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit != 0ull && (done.load(std::memory_order_acquire) & bit) != 0ull) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit != 0ull) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Asks for the largest shared-memory carveout for `kernel`, once per device.
// Every kernel of the library then runs with the same L1 / shared-memory
// split, so an SM moving from one kernel's CTAs to the next one's (dependent
// launches start CTAs as soon as SMs free up) does not first have to change
// its split.
cudaError_t prefer_max_shared(const void* kernel);

// Launches `kernel` on `stream` as a programmatic dependent of the work before
// it (see pdl_wait), optionally as clusters of `cluster_x` CTAs.
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       int cluster_x, Args... args) {
  const cudaError_t ce = prefer_max_shared(reinterpret_cast<const void*>(kernel));
  if (ce != cudaSuccess) return ce;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Driver entry point for tensor-map encoding, resolved once through the
// runtime (no link-time dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

}  // namespace dsa
