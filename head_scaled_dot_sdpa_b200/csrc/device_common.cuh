// Device helpers shared by the kernels: element conversion, status reporting and the
// per-batch resolution of lengths and causal offsets.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "internal.h"

namespace sdpa {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Records the first device-side error in the status word; later errors keep the first.
__device__ __forceinline__ void report(int* status, int code) {
  if (status) atomicCAS(status, kStatusOk, code);
}

// Range checks of the build compiled with SDPA_DEBUG_CHECKS (libsdpa_debug.so): SDPA_CHECKED(st,
// cond) is cond, and a false cond records SDPA_ERR_DEVICE_CHECK in the status word; the caller
// then skips (or clamps) the access. In the normal build it is the constant true, and the
// compiler removes the check.
__device__ __forceinline__ bool checked(int* status, bool ok) {
  if (!ok) report(status, SDPA_ERR_DEVICE_CHECK);
  return ok;
}
#ifdef SDPA_DEBUG_CHECKS
#define SDPA_CHECKED(status, cond) (::sdpa::checked((status), (cond)))
#else
#define SDPA_CHECKED(status, cond) (true)
#endif

// The dropout draw of scaled_dot_product_attention_with_weights (argument fdrop as dropout):
// SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) used as a counter-based generator. Its n-th
// output from state `seed` is splitmix64_mix(seed + n * kSplitMixGamma). The weights' row-major
// positions (b, h, i, j) are taken four at a time: group g = index / 4 gets output n = g + 1,
// and the weight at `index` takes 16-bit field index % 4 of it (lowest first) as u in
// [0, 2^16); it is kept when u >= ceil(p * 2^16). Consecutive groups differ by one gamma in
// the mixed state, so a run of groups costs one 64-bit add and one mix each.
constexpr unsigned long long kSplitMixGamma = 0x9e3779b97f4a7c15ULL;
__device__ __forceinline__ unsigned long long splitmix64_mix(unsigned long long z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}
// the state that gives group g's draw
__device__ __forceinline__ unsigned long long dropout_state(unsigned long long seed, unsigned long long group) {
  return seed + (group + 1) * kSplitMixGamma;
}
__device__ __forceinline__ unsigned long long dropout_group_draw(unsigned long long seed, unsigned long long group) {
  return splitmix64_mix(dropout_state(seed, group));
}
// bits f of the result: whether field f (f < 4) of r is kept
__device__ __forceinline__ uint32_t dropout_keep4(unsigned long long r, unsigned threshold) {
  return (uint32_t)(((unsigned)r & 0xFFFFu) >= threshold) | ((uint32_t)(((unsigned)(r >> 16) & 0xFFFFu) >= threshold) << 1) |
         ((uint32_t)(((unsigned)(r >> 32) & 0xFFFFu) >= threshold) << 2) |
         ((uint32_t)((unsigned)(r >> 48) >= threshold) << 3);
}

// Lengths, offsets: the arguments q_lengths, kv_lengths, q_offset and is_causal of
// NNlib.scaled_dot_product_attention. Out-of-range lengths are clamped and reported.
// With packed sequences (keywords q_segments / kv_segments, paragraph "Packed sequences") the
// b-th segment plays the part of batch element b, its lengths bounding q_lengths / kv_lengths.
__device__ __forceinline__ BatchInfo resolve_batch(const Problem& P, int b) {
  BatchInfo bi;
  bi.skip = false;
  int qseg = P.Lq, kseg = P.Lk;
  if (P.q_start) {
    bi.q0 = P.q_start[b];
    bi.k0 = P.kv_start[b];
    qseg = P.q_start[b + 1] - (int)bi.q0;
    kseg = P.kv_start[b + 1] - (int)bi.k0;
  } else {
    bi.q0 = (long long)b * P.Lq;
    bi.k0 = (long long)b * P.Lk;
  }
  bi.q_rows = qseg;
  int ql = qseg, kl = kseg;
  if (P.q_lengths) {
    ql = P.q_lengths[b];
    if (ql < 0 || ql > qseg) {
      report(P.status, SDPA_ERR_DEVICE_CHECK);
      ql = ql < 0 ? 0 : qseg;
    }
  }
  if (P.cache_index) {
    const int idx = P.cache_index[b];
    bi.skip = idx < 0 || idx > P.Lk - P.Lq;  // reported by the cache update
    kl = bi.skip ? 0 : idx + P.Lq;
  } else if (P.kv_lengths) {
    kl = P.kv_lengths[b];
  }
  if (kl < 0 || kl > kseg) {
    report(P.status, SDPA_ERR_DEVICE_CHECK);
    kl = kl < 0 ? 0 : kseg;
  }
  bi.q_len = ql;
  bi.kv_len = kl;
  if (P.causal == SDPA_CAUSAL_TOP_LEFT)
    bi.offset = P.q_offset ? P.q_offset[b] : P.q_offset_scalar;
  else if (P.causal == SDPA_CAUSAL_BOTTOM_RIGHT)
    bi.offset = kl - ql;
  else
    bi.offset = 0x3fffffff;  // no causal limit
  return bi;
}

// Bias element (key j, query i, head h, batch b), as float.
__device__ __forceinline__ float load_bias(const Problem& P, int b, int h, long long i,
                                           long long j) {
  const long long off = j * P.bs[0] + i * P.bs[1] + (long long)h * P.bs[2] + (long long)b * P.bs[3];
  switch (P.bias_dtype) {
    case SDPA_F16: return __half2float(static_cast<const __half*>(P.bias)[off]);
    case SDPA_BF16: return __bfloat162float(static_cast<const __nv_bfloat16*>(P.bias)[off]);
    default: return static_cast<const float*>(P.bias)[off];
  }
}

// Whether the boolean mask (dense, or its block classification) lets query i of head h see
// key j. The block classification, when present, takes precedence over the dense mask.
__device__ __forceinline__ bool mask_allows(const Problem& P, int b, int h, int i, int j) {
  if (P.bcls) {
    const int hm = P.bi_nheads == 1 ? 0 : h;
    const int qb = i / P.bi_bq, kb = j / P.bi_bk;
    const long long blk = ((long long)hm * P.bi_nqb + qb) * P.bi_nkb + kb;
    const uint8_t c = P.bcls[blk];
    if (c == SDPA_BLOCK_EMPTY) return false;
    if (c == SDPA_BLOCK_FULL) return true;
    const int words = P.bi_bk / 32;
    const int r = i - qb * P.bi_bq, cc = j - kb * P.bi_bk;
    const uint32_t w = P.bbits[(blk * P.bi_bq + r) * words + cc / 32];
    return (w >> (cc % 32)) & 1u;
  }
  if (P.mask) {
    const long long off = (long long)j * P.ms[0] + (long long)i * P.ms[1] +
                          (long long)h * P.ms[2] + (long long)b * P.ms[3];
    return P.mask[off] != 0;
  }
  return true;
}

}  // namespace sdpa
