// dsa_sparse_attn_noalloc: the sparse-attention step for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the layer:
// code that executes inside a pre-sized memory pool it must not grow, an
// inference runtime that hands kernels only the tensors of the graph it owns,
// or a plugin host that forbids allocation after start-up.  For them this
// entry point takes only the inputs and outputs.  The scratch that
// dsa_sparse_attn keeps in the caller's workspace (the per-slice partial
// outputs, maxima and sums of few-row launches) lives here in one file-scope
// device array of kNoAllocScratchBytes (10 MiB), which every GPU that loads
// the library holds until the process exits.  10 MiB covers every split the
// launch planner makes (at most about 9.3 MiB of partials); a launch that
// would need more is rejected with DSA_ERR_WORKSPACE before anything runs.
// The kernels are the CUDA-core attention kernels of the library; only where
// their scratch lives differs.
//
// The first call on a device looks up the array's device address (once per
// device, under a lock); make that first call before capturing a stream into
// a CUDA graph.  All calls share the one array: calls whose work overlaps on
// the GPU (two streams, or two threads on one device) race on it and must be
// serialised by the caller.
#include <mutex>

#include "../../include/dsa.h"
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(10) << 20;  // 10 MiB

// Partial results of the split launches; the whole array is overwritten by
// each call that uses it, so nothing in it has to start at zero.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array, looked up once per device with that device
// current (in host code the array's name is not a device address).
constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

cudaError_t scratch_for_current_device(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return cudaSuccess;
}

bool aligned16_na(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" DSA_API dsa_status dsa_sparse_attn_noalloc(const dsa_batch* batch, const uint16_t* q,
                                                      int H, const uint16_t* kv,
                                                      const int32_t* idx, int top_k,
                                                      float scale, float* out, float* lse,
                                                      void* stream) {
  // Same argument rules as dsa_sparse_attn.
  if (!batch || batch->B < 0 || batch->Nq < 0) return DSA_ERR_INVALID_ARG;
  if (batch->B == 0) return batch->Nq == 0 ? DSA_OK : DSA_ERR_INVALID_ARG;
  if (!batch->q_offsets || !batch->kv_offsets || !batch->ctx_lens || !batch->h_q_offsets ||
      !batch->h_kv_offsets || !batch->h_ctx_lens) {
    return DSA_ERR_INVALID_ARG;
  }
  if (batch->h_q_offsets[0] != 0 || batch->h_q_offsets[batch->B] != batch->Nq ||
      batch->h_kv_offsets[0] < 0) {
    return DSA_ERR_INVALID_ARG;
  }
  for (int i = 0; i < batch->B; ++i) {
    const int64_t nq = static_cast<int64_t>(batch->h_q_offsets[i + 1]) - batch->h_q_offsets[i];
    const int64_t cap = batch->h_kv_offsets[i + 1] - batch->h_kv_offsets[i];
    const int64_t L = batch->h_ctx_lens[i];
    if (nq < 0 || cap < 0 || L < 0 || nq > L || L > cap) return DSA_ERR_INVALID_ARG;
  }
  if (H < 1 || top_k < 1) return DSA_ERR_INVALID_ARG;
  if (H > kMaxHeads || top_k > kMaxTopK) return DSA_ERR_UNSUPPORTED;
  if (batch->Nq == 0) return DSA_OK;
  if (!q || !kv || !idx || !out) return DSA_ERR_INVALID_ARG;
  if (!aligned16_na(q) || !aligned16_na(kv) || !aligned16_na(idx) || !aligned16_na(out) ||
      (lse && !aligned16_na(lse))) {
    return DSA_ERR_UNSUPPORTED;
  }
  if (!isfinite(scale)) return DSA_ERR_INVALID_ARG;

  // The CUDA-core kernels and their split plan.
  const AttnPlan plan = attn_plan_core(batch->Nq, H, top_k, 148);
  if (attn_partial_bytes(batch->Nq, H, plan) > kNoAllocScratchBytes) return DSA_ERR_WORKSPACE;

  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return DSA_ERR_NOT_SM100;
  }
  if (major != 10 || minor != 0) return DSA_ERR_NOT_SM100;
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return DSA_ERR_CUDA;

  AttnArgs a;
  a.B = batch->B;
  a.Nq = batch->Nq;
  a.q_offsets = batch->q_offsets;
  a.kv_offsets = batch->kv_offsets;
  a.ctx_lens = batch->ctx_lens;
  a.q = q;
  a.H = H;
  a.kv = kv;
  a.idx = idx;
  a.top_k = top_k;
  a.scale = scale;
  a.out = out;
  a.lse = lse;
  a.part = static_cast<float*>(scratch);
  a.err = nullptr;  // the CUDA-core kernels never wait on a barrier
  a.idx_prefix = false;
  a.batch_ready = false;
  a.plan = plan;
  return launch_sparse_attn(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? DSA_OK
                                                                                   : DSA_ERR_CUDA;
}
