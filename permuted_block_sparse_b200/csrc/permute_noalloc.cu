// pbs_permute_noalloc: the key permutation for callers that cannot allocate.
//
// pbs_permute needs a small device workspace (the pooled proxy query, one
// fp32 vector of D per (batch, KV head)) that the caller allocates.  Some
// callers cannot do that at call time: a runtime whose device memory is
// entirely reserved up front by its own allocator, or a plugin interface that
// hands a kernel only its input and output buffers and no workspace slot.
// This entry point keeps that workspace in a fixed, file-scope device array
// instead, so the call itself allocates nothing.
//
// The array is part of the library image: every GPU that loads libpbs.so
// holds its 256 KiB until the process exits.  All calls on a device share it,
// so calls whose work overlaps on the GPU (different streams, no ordering
// between them) race on it and must not be issued.  The array keeps the last
// call's contents; every call overwrites the part it reads before reading it,
// so nothing has to be cleared.
#include <mutex>

#include "pbs_common.cuh"
#include "pbs_internal.h"

namespace {

// B * Hkv * D floats at most (e.g. 512 KV-head rows of D = 128).
constexpr int64_t kScratchFloats = 65536;

static __device__ __align__(256) float g_permute_scratch[kScratchFloats];

// The array's device address for the current device, looked up once per
// device with that device current.  In host code the symbol itself is only a
// host-side stand-in and must never be handed to a kernel.
float* scratch_for_current_device() {
  static std::mutex mu;
  static float* addr[128] = {nullptr};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<float*>(p);
  }
  return addr[dev];
}

}  // namespace

extern "C" int pbs_permute_noalloc(const pbs_tensor* Qt, const pbs_tensor* Kt, int blk, int seg,
                                   int n_sink, int32_t* perm, void* stream) {
  pbs::TensorDesc Q, K;
  int rc = pbs::api_validate_permute(Qt, Kt, blk, seg, n_sink, perm, &Q, &K);
  if (rc) return rc;
  if (K.B * K.H * K.D > kScratchFloats)
    return pbs::api_fail(PBS_ERR_CAPACITY,
                         "pbs_permute_noalloc: B*Hkv*D exceeds the 65536-float static scratch");
  float* qhat = scratch_for_current_device();
  if (!qhat) return pbs::api_fail(PBS_ERR_CUDA, "pbs_permute_noalloc: cannot resolve the static scratch");
  int* err = pbs::api_device_error_word();
  if (!err) return pbs::api_fail(PBS_ERR_CUDA, "cannot resolve the device error word");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = pbs::launch_pool_proxy_query(Q, static_cast<int>(K.H), blk, qhat, s);
  if (e != cudaSuccess) return pbs::api_fail(PBS_ERR_CUDA, cudaGetErrorString(e));
  e = pbs::launch_score_sort(K, seg, n_sink, qhat, perm, err, s);
  if (e != cudaSuccess) return pbs::api_fail(PBS_ERR_CUDA, cudaGetErrorString(e));
  return pbs::api_ok();
}
