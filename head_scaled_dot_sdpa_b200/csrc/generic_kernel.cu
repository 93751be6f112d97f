// Generic SIMT attention kernel: every semantic of NNlib.scaled_dot_product_attention (Flux.jl
// page "Neural Network primitives from NNlib.jl", sections "Arguments" and "Fused
// implementation") for any element type and head size, on the CUDA cores.
//
// It serves fp32 (where tensor-core TF32 would miss a 1e-5 tolerance) and the head sizes the
// tcgen05 prefill kernel does not cover. One warp owns one query row (b, i, h): lanes take 32
// keys at a time, each lane one key's dot product; the chunk's logits go through an online
// softmax (running max m and sum l, rescaling the output by exp(m_old - m_new)), and each lane
// accumulates the value dimensions e = lane, lane + 32, ... . Weights are never materialised.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device_common.cuh"

namespace sdpa {
namespace {

constexpr int kWarps = 4;
constexpr int kMaxDvPerLane = 8;  // dv <= 256

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
generic_attention_kernel(Problem P, const T* __restrict__ q, const T* __restrict__ k,
                         const T* __restrict__ v, T* __restrict__ out) {
  extern __shared__ float q_smem[];  // [kWarps][D]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long row = (long long)blockIdx.x * kWarps + warp;  // (b, i, h), h fastest
  const long long rows = (long long)P.B * P.Lq * P.H;
  if (row >= rows) return;
  const int h = (int)(row % P.H);
  const int i = (int)((row / P.H) % P.Lq);
  const int b = (int)(row / ((long long)P.H * P.Lq));
  const int D = P.D, Dv = P.Dv;

  // row (b, i, h) of a padded batch, or row i of packed sequence b (whose rows start at bi.q0;
  // rows past the sequence belong to the next one and are left alone)
  const BatchInfo bi = resolve_batch(P, b);
  if (i >= bi.q_rows) return;
  const long long qi = (bi.q0 + i) * P.H + h;
  if (bi.skip) {
    // decode with an out-of-range cache index (reported by the cache update): NaN rows
    T* orow = out + qi * Dv;
    for (int e = lane; e < Dv; e += 32) orow[e] = from_f32<T>(__int_as_float(0x7fc00000));
    return;
  }
  float* qs = q_smem + warp * D;
  const T* qrow = q + qi * D;
  for (int c = lane; c < D; c += 32) qs[c] = to_f32(qrow[c]);
  __syncwarp();

  T* orow = out + qi * Dv;
  if (i >= bi.q_len) {  // argument q_lengths: padding rows are zero
    for (int e = lane; e < Dv; e += 32) orow[e] = from_f32<T>(0.f);
    return;
  }
  const int g = h / P.group;  // GQA: contiguous groups of query heads share a K/V head
  long long jend = bi.kv_len;
  if (P.causal != SDPA_CAUSAL_NONE) {
    const long long lim = (long long)bi.offset + i + 1;  // keys j <= offset + i
    jend = lim < jend ? (lim < 0 ? 0 : lim) : jend;
  }

  float m = -INFINITY, l = 0.f;
  float o[kMaxDvPerLane];
#pragma unroll
  for (int t = 0; t < kMaxDvPerLane; ++t) o[t] = 0.f;

  for (long long j0 = 0; j0 < jend; j0 += 32) {
    const long long j = j0 + lane;
    float s = -INFINITY;
    if (j < jend && mask_allows(P, b, h, i, (int)j)) {
      const T* kr = k + ((bi.k0 + j) * P.Hkv + g) * D;
      float acc = 0.f;
      for (int c = 0; c < D; ++c) acc = fmaf(qs[c], to_f32(kr[c]), acc);
      s = acc * P.scale;
      if (P.bias) s += load_bias(P, b, h, i, j);
    }
    const float m_new = fmaxf(m, warp_max(s));
    if (m_new == -INFINITY) continue;  // nothing attended so far
    const float p = (s == -INFINITY) ? 0.f : expf(s - m_new);
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    l = l * alpha + warp_sum(p);
#pragma unroll
    for (int t = 0; t < kMaxDvPerLane; ++t) o[t] *= alpha;
    const int n = (int)((jend - j0) < 32 ? (jend - j0) : 32);
    for (int t = 0; t < n; ++t) {
      const float pt = __shfl_sync(0xffffffffu, p, t);
      if (pt == 0.f) continue;  // warp-uniform
      const T* vr = v + ((bi.k0 + j0 + t) * P.Hkv + g) * Dv;
#pragma unroll
      for (int u = 0; u < kMaxDvPerLane; ++u) {
        const int e = lane + 32 * u;
        if (e < Dv) o[u] = fmaf(pt, to_f32(vr[e]), o[u]);
      }
    }
    m = m_new;
  }

  // A query attending to no key is NaN (section "Fused implementation").
  const float inv = (l > 0.f) ? 1.f / l : __int_as_float(0x7fc00000);
#pragma unroll
  for (int u = 0; u < kMaxDvPerLane; ++u) {
    const int e = lane + 32 * u;
    if (e < Dv) orow[e] = from_f32<T>(l > 0.f ? o[u] * inv : inv);
  }
}

}  // namespace

cudaError_t launch_generic(const Problem& P, const void* q, const void* k, const void* v,
                           void* out, cudaStream_t stream) {
  const long long rows = (long long)P.B * P.Lq * P.H;
  if (rows == 0) return cudaSuccess;
  const dim3 grid((unsigned)((rows + kWarps - 1) / kWarps));
  const size_t smem = sizeof(float) * kWarps * P.D;
  switch (P.dtype) {
    case SDPA_F32:
      generic_attention_kernel<float><<<grid, kWarps * 32, smem, stream>>>(
          P, (const float*)q, (const float*)k, (const float*)v, (float*)out);
      break;
    case SDPA_F16:
      generic_attention_kernel<__half><<<grid, kWarps * 32, smem, stream>>>(
          P, (const __half*)q, (const __half*)k, (const __half*)v, (__half*)out);
      break;
    default:
      generic_attention_kernel<__nv_bfloat16><<<grid, kWarps * 32, smem, stream>>>(
          P, (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
          (__nv_bfloat16*)out);
      break;
  }
  return cudaGetLastError();
}

}  // namespace sdpa
