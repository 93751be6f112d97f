// Decoding with a KV cache without a caller-supplied workspace.
//
// Some callers of this library cannot allocate device memory: a plug-in hosted by a framework
// that owns every device allocation and gives plug-ins no allocator, or a latency-critical
// decode loop that must never block on (or fail in) the driver's allocator in the middle of a
// run. They cannot provide the workspace sdpa_decode_with_cache needs for its split-KV
// partials. sdpa_decode_with_cache_static gives them the same operation with the scratch in a
// fixed-size array that lives in the library itself: SDPA_STATIC_SCRATCH_BYTES (40 MiB) of
// device memory, which every GPU that loads the library holds until the process exits.
//
// The array's name is only a host-side stand-in in host code, not a device address; its device
// address is looked up once per device with cudaGetSymbolAddress, with that device current, and
// then passed to the kernels. The first call on each device does that lookup. The first 256
// bytes of the array are the status word area of the workspace layout; sdpa_read_static_status
// reads and clears it.
#include <cstdio>
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kScratchBytes = SDPA_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// The array's device address on the current device (looked up on first use), or null with the
// error message set.
void* scratch_for_current_device(bool look_up, sdpa_status* st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    sdpa::set_last_error("cudaGetDevice failed or device ordinal out of range");
    *st = SDPA_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev] && look_up) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess || !ptr) {
      char msg[256];
      snprintf(msg, sizeof(msg), "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
      sdpa::set_last_error(msg);
      *st = SDPA_ERR_CUDA;
      return nullptr;
    }
    g_scratch_ptr[dev] = ptr;
  }
  *st = SDPA_OK;
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" sdpa_status sdpa_decode_with_cache_static(const sdpa_params* p, const void* q, const void* k_new,
                                                     const void* v_new, void* k_cache, void* v_cache,
                                                     const int32_t* cache_index, void* out,
                                                     struct CUstream_st* stream) {
  // size check first: nothing is set up or launched for a call that cannot fit
  const size_t need = sdpa_workspace_size(p);
  if (need == 0) return sdpa_decode_with_cache(p, q, k_new, v_new, k_cache, v_cache, cache_index, out,
                                               nullptr, 0, stream);  // reports the invalid argument
  if (need > kScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "this decode call needs %zu bytes of scratch; the static scratch holds %zu bytes "
             "(use sdpa_decode_with_cache with a larger workspace)",
             need, kScratchBytes);
    sdpa::set_last_error(msg);
    return SDPA_ERR_WORKSPACE;
  }
  sdpa_status st = SDPA_OK;
  void* scratch = scratch_for_current_device(true, &st);
  if (!scratch) return st;
  // the array keeps the previous call's contents: the status word is cleared once the
  // arguments have passed every check, before the kernels that may write it
  return sdpa::decode_with_cache(p, q, k_new, v_new, k_cache, v_cache, cache_index, out, scratch, kScratchBytes,
                                 (cudaStream_t)stream, true);
}

extern "C" sdpa_status sdpa_read_static_status(struct CUstream_st* stream) {
  sdpa_status st = SDPA_OK;
  void* scratch = scratch_for_current_device(false, &st);
  if (st != SDPA_OK) return st;
  if (!scratch) return SDPA_OK;  // no static call has run on this device
  return sdpa_read_device_status(scratch, stream);
}
