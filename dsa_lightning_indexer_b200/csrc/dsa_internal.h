// Host-side interfaces between the C ABI layer (dsa_api.cu) and the kernel
// translation units.  Arguments here are already validated.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace dsa {

struct IndexerArgs {
  int B;
  const int32_t* h_q_offsets;   // host mirrors of the batch
  const int64_t* h_kv_offsets;
  const int32_t* h_ctx_lens;
  int Nq;
  int64_t cache_rows;   // rows of k_idx (kv_offsets[B])
  const uint16_t* q_idx;
  const float* w;
  const uint16_t* k_idx;
  float* scores;
  int64_t ld;
  unsigned* err;
  int num_sms;
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
};
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream);

struct AttnArgs {
  int B;
  int Nq;
  const int32_t* q_offsets;   // device
  const int64_t* kv_offsets;  // device
  const uint16_t* q;
  int H;
  const uint16_t* kv;
  const int32_t* idx;
  int top_k;
  float scale;
  float* out;
  float* lse;
  float* part;        // split partials (workspace), may be null when n_split == 1
  int n_split;
  int num_sms;
};
// Number of key splits the attention launch uses for this shape.
int attn_num_splits(int Nq, int H, int top_k, int num_sms);
size_t attn_partial_bytes(int Nq, int H, int n_split);
cudaError_t launch_sparse_attn(const AttnArgs& a, cudaStream_t stream);

// Driver entry point for tensor-map encoding, resolved once through the
// runtime (no link-time dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

}  // namespace dsa
