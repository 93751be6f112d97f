// Writing new key/value rows into a KV cache at a per-sequence index (Keras issue
// "MultiHeadAttention is missing a position_bias call argument": cache_update_index; Flax
// discussion on decode=True: cached_key / cached_value of shape (batch, len, heads, head_dim)).
//
//   cache[b][index[b] + t][:][:] = new[b][t][:][:]     for t < n_new
//
// The index lives on the device; a sequence whose index is out of range is skipped and the
// status word records SDPA_ERR_DEVICE_CHECK. The copy moves 16-byte words when every row is a
// whole number of them (the usual case: nkvheads * head_dim * 2 bytes), else elements.
#include "device_common.cuh"

namespace sdpa {
namespace {

template <typename W>
__global__ void cache_update_kernel(W* __restrict__ kc, W* __restrict__ vc,
                                    const W* __restrict__ kn, const W* __restrict__ vn,
                                    int row_words, int n_new, int capacity, int B,
                                    const int32_t* __restrict__ index, int* status) {
  const int b = blockIdx.y;
  const int idx = index[b];
  if (idx < 0 || idx > capacity - n_new) {
    if (threadIdx.x == 0 && blockIdx.x == 0) report(status, SDPA_ERR_DEVICE_CHECK);
    return;
  }
  const long long per_batch = (long long)n_new * row_words;
  const long long dst0 = ((long long)b * capacity + idx) * row_words;
  const long long src0 = (long long)b * per_batch;
  for (long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x; w < per_batch;
       w += (long long)gridDim.x * blockDim.x) {
    if (kc) kc[dst0 + w] = kn[src0 + w];
    if (vc) vc[dst0 + w] = vn[src0 + w];
  }
}

}  // namespace

cudaError_t launch_cache_update(void* k_cache, void* v_cache, const void* k_new,
                                const void* v_new, int esize, int d, int Hkv, int n_new,
                                int capacity, int B, const int32_t* index, int* status,
                                cudaStream_t stream) {
  if (B == 0 || n_new == 0) return cudaSuccess;
  const long long row_bytes = (long long)Hkv * d * esize;
  auto aligned16 = [](const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  const bool vec = (row_bytes % 16 == 0) && aligned16(k_cache) && aligned16(v_cache) &&
                   aligned16(k_new) && aligned16(v_new);
  const int threads = 256;
  if (vec) {
    const int row_words = (int)(row_bytes / 16);
    const long long per_batch = (long long)n_new * row_words;
    unsigned gx = (unsigned)((per_batch + threads - 1) / threads);
    if (gx > 1024) gx = 1024;
    cache_update_kernel<uint4><<<dim3(gx, B), threads, 0, stream>>>(
        (uint4*)k_cache, (uint4*)v_cache, (const uint4*)k_new, (const uint4*)v_new, row_words,
        n_new, capacity, B, index, status);
  } else {
    const int row_words = (int)(row_bytes / esize);
    const long long per_batch = (long long)n_new * row_words;
    unsigned gx = (unsigned)((per_batch + threads - 1) / threads);
    if (gx > 1024) gx = 1024;
    if (esize == 4)
      cache_update_kernel<uint32_t><<<dim3(gx, B), threads, 0, stream>>>(
          (uint32_t*)k_cache, (uint32_t*)v_cache, (const uint32_t*)k_new, (const uint32_t*)v_new,
          row_words, n_new, capacity, B, index, status);
    else
      cache_update_kernel<uint16_t><<<dim3(gx, B), threads, 0, stream>>>(
          (uint16_t*)k_cache, (uint16_t*)v_cache, (const uint16_t*)k_new, (const uint16_t*)v_new,
          row_words, n_new, capacity, B, index, status);
  }
  return cudaGetLastError();
}

}  // namespace sdpa
