// sq_noalloc.cu -- the split decode step with its staging buffer in a fixed, library-owned
// device array, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: serving engines that reserve the whole device memory for
// their own allocator at start-up and forbid allocations behind its back, and embedded or
// real-time hosts whose memory plan is fixed before the first request. For them this file keeps
// the scratch state of sq_decode_step_split (fp32, one d_k x d_v tile per request-head) in a
// static device array of kStagingBytes, which every GPU that loads libsq holds until the process
// exits.
#include <cuda_runtime.h>

#include "sq.h"
#include "sq_internal.h"

namespace {

constexpr size_t kStagingBytes = size_t(32) << 20;  // 32 MiB: 512 request-heads at d = 128

static __device__ __align__(256) unsigned char g_staging[kStagingBytes];

// Device address of g_staging on the current device, looked up on every call (the lookup
// allocates nothing and costs little; a cached address would go stale if the device's context
// were torn down and created again). In host code `g_staging` names a host-side stand-in, not
// device memory, so it is never passed to a kernel itself. The first lookup on a device may
// load the library's module there, which is why the first call should come before any stream
// capture.
sq_status staging_on_current_device(float** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_staging) != cudaSuccess || !p) return SQ_ERR_CUDA;
  *out = static_cast<float*>(p);
  return SQ_OK;
}

}  // namespace

extern "C" sq_status sq_decode_step_split_static(sq_pool* pool, const int32_t* slot_idx,
                                                 int32_t batch, const void* q, const void* k,
                                                 const void* v, const float* alpha,
                                                 const float* beta, float* out, void* stream) {
  if (!pool || batch < 0) return SQ_ERR_INVALID_ARG;
  if (batch == 0) return SQ_OK;
  int H = 0, dk = 0, dv = 0;
  sq::pool_dims(pool, &H, &dk, &dv);
  if ((size_t)batch * (size_t)H * (size_t)dk * (size_t)dv * sizeof(float) > kStagingBytes)
    return SQ_ERR_INVALID_ARG;
  float* staging = nullptr;
  const sq_status s = staging_on_current_device(&staging);
  if (s != SQ_OK) return s;
  // both halves on the caller's stream: the staging array is ready for the next call once
  // this stream reaches it
  return sq_decode_step_split(pool, slot_idx, batch, q, k, v, alpha, beta, out, staging, stream,
                              stream);
}
