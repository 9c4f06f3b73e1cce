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
// device, under a lock).  Under lazy module loading (the CUDA 12 default) that
// lookup is also when the module holding the array is loaded, so the 10 MiB
// are committed then and the lookup can fail in a device whose memory is
// already full: make the first call at start-up, before memory fills up and
// before any stream is captured into a CUDA graph.  All calls share the one
// array: calls whose work overlaps on the GPU (two streams, or two threads on
// one device) race on it and must be serialised by the caller.
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
    if (e != cudaSuccess) {
      cudaGetLastError();  // leave no sticky error for the caller's next CUDA call
      return e;
    }
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" DSA_API dsa_status dsa_sparse_attn_noalloc(const dsa_batch* batch, const uint16_t* q,
                                                      int H, const uint16_t* kv,
                                                      const int32_t* idx, int top_k,
                                                      float scale, float* out, float* lse,
                                                      void* stream) {
  // Same argument rules as dsa_sparse_attn (the same validation helpers).
  BatchInfo info;
  dsa_status st = check_batch(batch, &info);
  if (st == DSA_OK) st = check_heads(H);
  if (st == DSA_OK) st = check_topk(top_k);
  if (st != DSA_OK || batch->Nq == 0) return st;
  const void* ptrs[] = {q, kv, idx, out};
  for (const void* p : ptrs) {
    if ((st = check_ptr(p)) != DSA_OK) return st;
  }
  if (lse && (st = check_ptr(lse)) != DSA_OK) return st;
  if (!isfinite(scale)) return DSA_ERR_INVALID_ARG;
  int sms = 0;
  if ((st = check_device(&sms)) != DSA_OK) return st;

  // The CUDA-core kernels and their split plan for this device's SM count.
  const AttnPlan plan = attn_plan_core(batch->Nq, H, top_k, sms);
  if (attn_partial_bytes(batch->Nq, H, plan) > kNoAllocScratchBytes) return DSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return DSA_ERR_CUDA;

  AttnArgs a;
  a.B = batch->B;
  a.Nq = batch->Nq;
  a.q_offsets = batch->q_offsets;
  a.cache.kv_offsets = batch->page_size > 0 ? nullptr : batch->kv_offsets;
  a.cache.block_table = batch->page_size > 0 ? batch->block_table : nullptr;
  a.cache.max_blocks = batch->page_size > 0 ? batch->max_blocks : 0;
  a.cache.page_shift = info.page_shift;
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
  a.cache_rows = info.cache_rows;
  a.plan = plan;
  return launch_sparse_attn(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? DSA_OK
                                                                                   : DSA_ERR_CUDA;
}
