// The gradient of the fused implementation (Flux.jl page "Neural Network primitives from
// NNlib.jl", entry scaled_dot_product_attention, paragraph "Fused implementation"): with
// respect to query, key, value and scale. The weights are recomputed from the logits and
// never materialized. A query that attends to no key (NaN output) takes no part, and neither
// does a query past q_lengths (its output is a constant zero).
//
// For the loss sum(dout * out) and one query row i with weights w_j over its attended keys:
//   dv_j += w_j dout_i,   dw_j = dout_i . v_j,   dx_j = w_j (dw_j - delta_i),
//   delta_i = sum_j w_j dw_j = dout_i . out_i,
//   dq_i = scale sum_j dx_j k_j,   dk_j += scale dx_j q_i,   dscale += sum_j dx_j (q_i . k_j).
//
// Three SIMT kernels on the CUDA cores, fp32 throughout (any element type, head sizes up to
// 256, every masking argument except a bias):
//  1. row statistics: per query row, the log-sum-exp of its scaled logits and delta_i
//     (+inf log-sum-exp marks a row that takes no part);
//  2. dq: one warp per query row, lanes over 32 keys at a time (the forward SIMT kernel's
//     walk), dscale reduced per block;
//  3. dk and dv: one warp per key row of a key/value head, lanes over 32 query rows at a time
//     of every query head of its group, so each dk / dv row is written once, without atomics.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device_common.cuh"

namespace sdpa {
namespace {

constexpr int kWarps = 4;
constexpr int kMaxPerLane = 8;  // head sizes up to 256

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

// Keys a query row may attend before the mask: j < kv_len and, with is_causal, j <= offset + i.
__device__ __forceinline__ long long key_end(const Problem& P, const BatchInfo& bi, int i) {
  long long jend = bi.kv_len;
  if (P.causal != SDPA_CAUSAL_NONE) {
    const long long lim = (long long)bi.offset + i + 1;
    jend = lim < jend ? (lim < 0 ? 0 : lim) : jend;
  }
  return jend;
}

// Query row (b, i, h) of a warp from its flat index (h fastest), as the forward kernel does.
struct Row {
  int b, i, h;
};
__device__ __forceinline__ Row row_of(const Problem& P, long long row) {
  Row r;
  r.h = (int)(row % P.H);
  r.i = (int)((row / P.H) % P.Lq);
  r.b = (int)(row / ((long long)P.H * P.Lq));
  return r;
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
bwd_row_stats_kernel(Problem P, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ out,
                     const T* __restrict__ dout, float* __restrict__ lse, float* __restrict__ delta,
                     float* dscale) {
  extern __shared__ float smem[];  // [kWarps][D]
  if (dscale && blockIdx.x == 0 && threadIdx.x == 0) *dscale = 0.f;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long row = (long long)blockIdx.x * kWarps + warp;
  if (row >= (long long)P.B * P.Lq * P.H) return;
  const Row r = row_of(P, row);
  const BatchInfo bi = resolve_batch(P, r.b);
  if (r.i >= bi.q_rows) return;
  const long long qi = (bi.q0 + r.i) * P.H + r.h;
  if (r.i >= bi.q_len) {  // padding row: constant zero output, no part in the gradient
    if (lane == 0) {
      lse[qi] = INFINITY;
      delta[qi] = 0.f;
    }
    return;
  }
  const int D = P.D, Dv = P.Dv, g = r.h / P.group;
  float* qs = smem + warp * D;
  for (int c = lane; c < D; c += 32) qs[c] = to_f32(q[qi * D + c]);
  __syncwarp();
  const long long jend = key_end(P, bi, r.i);
  float m = -INFINITY, l = 0.f;
  for (long long j0 = 0; j0 < jend; j0 += 32) {
    const long long j = j0 + lane;
    float s = -INFINITY;
    if (j < jend && mask_allows(P, r.b, r.h, r.i, (int)j)) {
      const T* kr = k + ((bi.k0 + j) * P.Hkv + g) * D;
      float acc = 0.f;
      for (int c = 0; c < D; ++c) acc = fmaf(qs[c], to_f32(kr[c]), acc);
      s = acc * P.scale;
    }
    const float m_new = fmaxf(m, warp_max(s));
    if (m_new == -INFINITY) continue;
    const float p = (s == -INFINITY) ? 0.f : expf(s - m_new);
    l = l * ((m == -INFINITY) ? 0.f : expf(m - m_new)) + warp_sum(p);
    m = m_new;
  }
  float dd = 0.f;
  for (int e = lane; e < Dv; e += 32) dd = fmaf(to_f32(dout[qi * Dv + e]), to_f32(out[qi * Dv + e]), dd);
  dd = warp_sum(dd);
  if (lane == 0) {
    lse[qi] = (l > 0.f) ? m + logf(l) : INFINITY;  // no attended key: no part in the gradient
    delta[qi] = dd;
  }
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
bwd_dq_kernel(Problem P, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
              const T* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ delta,
              T* __restrict__ dq, float* dscale) {
  extern __shared__ float smem[];  // [kWarps][D + Dv]
  __shared__ float block_ds[kWarps];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int D = P.D, Dv = P.Dv;
  const long long row = (long long)blockIdx.x * kWarps + warp;
  float ds_acc = 0.f;
  if (row < (long long)P.B * P.Lq * P.H) {
    const Row r = row_of(P, row);
    const BatchInfo bi = resolve_batch(P, r.b);
    if (r.i < bi.q_rows) {
      const long long qi = (bi.q0 + r.i) * P.H + r.h;
      const float L = lse[qi], dl = delta[qi];
      float acc[kMaxPerLane];
#pragma unroll
      for (int u = 0; u < kMaxPerLane; ++u) acc[u] = 0.f;
      if (L != INFINITY) {
        const int g = r.h / P.group;
        float* qs = smem + warp * (D + Dv);
        float* ds_row = qs + D;
        for (int c = lane; c < D; c += 32) qs[c] = to_f32(q[qi * D + c]);
        for (int e = lane; e < Dv; e += 32) ds_row[e] = to_f32(dout[qi * Dv + e]);
        __syncwarp();
        const long long jend = key_end(P, bi, r.i);
        for (long long j0 = 0; j0 < jend; j0 += 32) {
          const long long j = j0 + lane;
          float dx = 0.f;
          if (j < jend && mask_allows(P, r.b, r.h, r.i, (int)j)) {
            const T* kr = k + ((bi.k0 + j) * P.Hkv + g) * D;
            const T* vr = v + ((bi.k0 + j) * P.Hkv + g) * Dv;
            float dot = 0.f, dw = 0.f;
            for (int c = 0; c < D; ++c) dot = fmaf(qs[c], to_f32(kr[c]), dot);
            for (int e = 0; e < Dv; ++e) dw = fmaf(ds_row[e], to_f32(vr[e]), dw);
            const float w = expf(dot * P.scale - L);
            dx = w * (dw - dl);
            ds_acc = fmaf(dx, dot, ds_acc);
          }
          const int n = (int)((jend - j0) < 32 ? (jend - j0) : 32);
          for (int t = 0; t < n; ++t) {
            const float dxt = __shfl_sync(0xffffffffu, dx, t);
            if (dxt == 0.f) continue;  // warp-uniform
            const T* kr = k + ((bi.k0 + j0 + t) * P.Hkv + g) * D;
#pragma unroll
            for (int u = 0; u < kMaxPerLane; ++u) {
              const int c = lane + 32 * u;
              if (c < D) acc[u] = fmaf(dxt, to_f32(kr[c]), acc[u]);
            }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kMaxPerLane; ++u) {
        const int c = lane + 32 * u;
        if (c < D) dq[qi * D + c] = from_f32<T>(acc[u] * P.scale);
      }
    }
  }
  // dscale: one atomic per block
  ds_acc = warp_sum(ds_acc);
  if (lane == 0) block_ds[warp] = ds_acc;
  __syncthreads();
  if (dscale && threadIdx.x == 0) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += block_ds[w];
    if (t != 0.f) atomicAdd(dscale, t);
  }
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
bwd_dkdv_kernel(Problem P, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const T* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ delta,
                T* __restrict__ dk, T* __restrict__ dv) {
  extern __shared__ float smem[];  // [kWarps][D + Dv]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int D = P.D, Dv = P.Dv;
  const long long row = (long long)blockIdx.x * kWarps + warp;  // (b, j, g), g fastest
  if (row >= (long long)P.B * P.Lk * P.Hkv) return;
  const int g = (int)(row % P.Hkv);
  const int j = (int)((row / P.Hkv) % P.Lk);
  const int b = (int)(row / ((long long)P.Hkv * P.Lk));
  const BatchInfo bi = resolve_batch(P, b);
  const long long kj = (bi.k0 + j) * P.Hkv + g;
  if (P.q_start && j >= P.kv_start[b + 1] - (int)bi.k0) return;  // past a packed sequence
  float ak[kMaxPerLane], av[kMaxPerLane];
#pragma unroll
  for (int u = 0; u < kMaxPerLane; ++u) ak[u] = av[u] = 0.f;
  if (j < bi.kv_len) {
    float* ks = smem + warp * (D + Dv);
    float* vs = ks + D;
    for (int c = lane; c < D; c += 32) ks[c] = to_f32(k[kj * D + c]);
    for (int e = lane; e < Dv; e += 32) vs[e] = to_f32(v[kj * Dv + e]);
    __syncwarp();
    // queries that may see key j: i < q_len and, with is_causal, i >= j - offset
    long long i_begin = 0;
    if (P.causal != SDPA_CAUSAL_NONE) i_begin = (long long)j - bi.offset;
    if (i_begin < 0) i_begin = 0;
    for (int h = g * P.group; h < (g + 1) * P.group; ++h) {
      for (long long i0 = i_begin; i0 < bi.q_len; i0 += 32) {
        const long long i = i0 + lane;
        float w = 0.f, dx = 0.f;
        const long long qi = (bi.q0 + i) * P.H + h;
        if (i < bi.q_len && mask_allows(P, b, h, (int)i, j)) {
          const float L = lse[qi];
          if (L != INFINITY) {
            const T* qr = q + qi * D;
            const T* dr = dout + qi * Dv;
            float dot = 0.f, dw = 0.f;
            for (int c = 0; c < D; ++c) dot = fmaf(to_f32(qr[c]), ks[c], dot);
            for (int e = 0; e < Dv; ++e) dw = fmaf(to_f32(dr[e]), vs[e], dw);
            w = expf(dot * P.scale - L);
            dx = w * (dw - delta[qi]);
          }
        }
        const int n = (int)((bi.q_len - i0) < 32 ? (bi.q_len - i0) : 32);
        for (int t = 0; t < n; ++t) {
          const float wt = __shfl_sync(0xffffffffu, w, t);
          const float dxt = __shfl_sync(0xffffffffu, dx, t);
          if (wt == 0.f && dxt == 0.f) continue;  // warp-uniform
          const long long qt = (bi.q0 + i0 + t) * P.H + h;
#pragma unroll
          for (int u = 0; u < kMaxPerLane; ++u) {
            const int c = lane + 32 * u;
            if (c < D) ak[u] = fmaf(dxt, to_f32(q[qt * D + c]), ak[u]);
            if (c < Dv) av[u] = fmaf(wt, to_f32(dout[qt * Dv + c]), av[u]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kMaxPerLane; ++u) {
    const int c = lane + 32 * u;
    if (c < D) dk[kj * D + c] = from_f32<T>(ak[u] * P.scale);
    if (c < Dv) dv[kj * Dv + c] = from_f32<T>(av[u]);
  }
}

template <typename T>
cudaError_t launch_t(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                     const void* dout, void* dq, void* dk, void* dv, float* dscale, float* lse, float* delta,
                     cudaStream_t stream) {
  const long long qrows = (long long)P.B * P.Lq * P.H, krows = (long long)P.B * P.Lk * P.Hkv;
  const dim3 gq((unsigned)((qrows + kWarps - 1) / kWarps)), gk((unsigned)((krows + kWarps - 1) / kWarps));
  if (qrows > 0) {
    bwd_row_stats_kernel<T><<<gq, kWarps * 32, sizeof(float) * kWarps * P.D, stream>>>(
        P, (const T*)q, (const T*)k, (const T*)out, (const T*)dout, lse, delta, dscale);
    bwd_dq_kernel<T><<<gq, kWarps * 32, sizeof(float) * kWarps * (P.D + P.Dv), stream>>>(
        P, (const T*)q, (const T*)k, (const T*)v, (const T*)dout, lse, delta, (T*)dq, dscale);
  }
  if (krows > 0)
    bwd_dkdv_kernel<T><<<gk, kWarps * 32, sizeof(float) * kWarps * (P.D + P.Dv), stream>>>(
        P, (const T*)q, (const T*)k, (const T*)v, (const T*)dout, lse, delta, (T*)dk, (T*)dv);
  return cudaGetLastError();
}

}  // namespace

size_t backward_workspace_bytes(const Problem& P) {
  const long long rows = P.q_start ? (long long)P.Lq_total * P.H : (long long)P.B * P.Lq * P.H;
  return (size_t)rows * 2 * sizeof(float) + 256;
}

cudaError_t launch_backward(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                            const void* dout, void* dq, void* dk, void* dv, float* dscale, void* ws,
                            cudaStream_t stream) {
  const long long rows = P.q_start ? (long long)P.Lq_total * P.H : (long long)P.B * P.Lq * P.H;
  float* lse = static_cast<float*>(ws);
  float* delta = lse + ((rows + 63) / 64) * 64;
  switch (P.dtype) {
    case SDPA_F32: return launch_t<float>(P, q, k, v, out, dout, dq, dk, dv, dscale, lse, delta, stream);
    case SDPA_F16: return launch_t<__half>(P, q, k, v, out, dout, dq, dk, dv, dscale, lse, delta, stream);
    default: return launch_t<__nv_bfloat16>(P, q, k, v, out, dout, dq, dk, dv, dscale, lse, delta, stream);
  }
}

}  // namespace sdpa
