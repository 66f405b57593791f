// seer_sparse_decode_noalloc: the sparse decode for callers that must not
// allocate device memory.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: a
// serving engine that reserved all free HBM for its KV-cache pool up front,
// a plugin inside a host application that owns every allocation, or a hot
// loop where cudaMalloc's implicit device synchronisation (and its failure
// modes under memory pressure) are not acceptable.  This entry point keeps
// the split partials and arrival counters in a fixed scratch array that is
// part of the library image instead, so the caller passes only inputs and
// outputs.
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes
// (8 MiB).  Every GPU that loads the library holds it until the process
// exits, and every call on a device shares it, so calls that overlap on the
// GPU (different streams, or different host threads) race on it and must be
// serialised by the caller.  Host code cannot use the array's name as a
// device address (on the host it names a stand-in object): the device address
// is looked up with cudaGetSymbolAddress, once per device, by the first call
// made while that device is current; make that first call before any stream
// capture.  The looked-up address is kept for the life of the process, so
// calls after cudaDeviceReset (which unloads the library's device image) are
// not supported.  Each call clears the counters it relies on (an async memset
// on the caller's stream) because the array keeps whatever the previous call
// left; a call rejected by its argument checks enqueues nothing, not even that
// memset.
#include <stdio.h>

#include <mutex>

#include "seer.h"
#include "seer_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of the scratch array on the current device (looked up once per device).
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

seer_status cuda_error(cudaError_t e, const char* what) {
  char buf[256];
  snprintf(buf, sizeof(buf), "seer_sparse_decode_noalloc: %s: %s", what, cudaGetErrorString(e));
  return (seer_status)seer::set_last_error(SEER_ERR_CUDA, buf);
}

}  // namespace

extern "C" seer_status seer_sparse_decode_noalloc(const seer_dims_t* dims, const void* q, const seer_kv_t* k,
                                                  const seer_kv_t* v, const int32_t* block_idx,
                                                  const int32_t* block_cnt, const int32_t* seqlens,
                                                  int32_t capacity, int32_t num_split, void* out, float* lse_out,
                                                  int32_t* err_word, void* stream) {
  if (!dims) return (seer_status)seer::set_last_error(SEER_ERR_INVALID_ARG, "dims is NULL");
  if (capacity < 1) return (seer_status)seer::set_last_error(SEER_ERR_INVALID_ARG, "capacity must be >= 1");
  if (num_split < -1) return (seer_status)seer::set_last_error(SEER_ERR_INVALID_ARG, "num_split must be >= -1");
  const int32_t ns = num_split;
  const size_t need = seer_sparse_decode_workspace_bytes(dims, capacity, ns);
  if (need > kNoAllocScratchBytes) {
    char buf[320];
    snprintf(buf, sizeof(buf),
             "seer_sparse_decode_noalloc: %d splits need %zu bytes of scratch, more than the fixed %zu-byte "
             "array; use fewer splits, or seer_sparse_decode with a caller workspace",
             (int)ns, need, kNoAllocScratchBytes);
    return (seer_status)seer::set_last_error(SEER_ERR_CAPACITY, buf);
  }
  void* scratch = nullptr;
  if (need > 0) {
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress");
  }
  // every argument check of seer_sparse_decode runs before anything is enqueued
  seer::DecodeLaunch L;
  const seer_status st = seer::prepare_sparse_decode(dims, q, k, v, block_idx, block_cnt, seqlens, capacity, ns,
                                                     scratch, need > 0 ? kNoAllocScratchBytes : 0, out, lse_out,
                                                     err_word, &L);
  if (st != SEER_OK) return st;
  if (L.need > 0) {
    // the arrival counters open the workspace layout (B * Hkv int32) and must start at zero
    const size_t counters = (size_t)dims->batch * dims->num_kv_heads * sizeof(int32_t);
    cudaError_t e = cudaMemsetAsync(scratch, 0, counters, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_error(e, "clearing the arrival counters");
  }
  return seer::launch_prepared_decode(L, static_cast<cudaStream_t>(stream));
}
