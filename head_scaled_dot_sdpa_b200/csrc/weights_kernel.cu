// scaled_dot_product_attention_with_weights with fdrop as dropout (Flux.jl page "Neural Network
// primitives from NNlib.jl", entry scaled_dot_product_attention: "See also", the argument fdrop,
// and the materialized implementation of the paragraph "Fused implementation"). The weights
// w_ij = softmax_j(scale q_i.k_j + bias_ij, masked) are written out (after the dropout, which
// keeps a weight with probability 1 - p and divides it by 1 - p), and out_i = sum_j w'_ij v_j.
//
// Layout of the weights: the page's (kv_len, q_len, nheads, batch), row-major
// [batch][nheads][q_len][kv_len], in the input type. A row with no attended key has NaN weights
// and output; a row past q_lengths has zero weights and output.
//
// The dropout draw is counter-based (SplitMix64, device_common.cuh): the weights' row-major
// positions are taken four at a time, group g = index / 4 gets the generator's output g + 1
// from state seed, and the weight at `index` takes the 16-bit field number index % 4 of it
// (lowest first) as u in [0, 2^16); it is kept when u >= ceil(p * 2^16), an integer
// comparison.
//
// Two kernels:
//  - weights_mma_kernel (bf16/fp16, head_dim = v_head_dim = 64 or 128): one CTA per
//    (64 queries, head, batch), 4 warps of 16 rows on mma.sync tiles. Pass 1 over the key
//    tiles gives the row log-sum-exp. Pass 2 computes the weights, stores them, and
//    accumulates out += w' V.
//  - weights_simt_kernel (any type and head size): one warp per query row, lanes over keys.
#include "mma_tiles.cuh"

namespace sdpa {
namespace {

using namespace tiles;

constexpr int kRows = 64;  // query rows per CTA
constexpr int kKeys = 64;  // keys per tile

// Whether the dropout keeps the weight at row-major position `index` (threshold =
// ceil(p * 2^16)).
__device__ __forceinline__ bool keep(unsigned long long seed, unsigned long long index, unsigned threshold) {
  return (dropout_keep4(dropout_group_draw(seed, index >> 2), threshold) >> (index & 3)) & 1u;
}

// The logit of (i, j) in log2 units: (scale q.k + bias) * log2(e), from the raw dot product.
__device__ __forceinline__ float logit2(const Problem& P, int b, int h, int i, int j, float dot) {
  float x = dot * P.scale;
  if (P.bias) x += load_bias(P, b, h, i, j);
  return x * kLog2e;
}

template <typename T> __device__ __forceinline__ T nan_of();
template <> __device__ __forceinline__ float nan_of<float>() { return __int_as_float(0x7fc00000); }
template <> __device__ __forceinline__ __half nan_of<__half>() { return __float2half(__int_as_float(0x7fc00000)); }
template <> __device__ __forceinline__ __nv_bfloat16 nan_of<__nv_bfloat16>() {
  return __float2bfloat16(__int_as_float(0x7fc00000));
}

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
weights_mma_kernel(Problem P, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   T* __restrict__ out, T* __restrict__ weights, double drop_p, unsigned long long seed) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kTileBytes = kRows * D * 2;
  const Tile<D> tq{su32(smem)};
  const Tile<D> tk[2] = {{su32(smem + kTileBytes)}, {su32(smem + 2 * kTileBytes)}};
  const Tile<D> tv[2] = {{su32(smem + 3 * kTileBytes)}, {su32(smem + 4 * kTileBytes)}};
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, gq = lane / 4, tq4 = lane % 4;
  const int h = blockIdx.y, b = blockIdx.z, i0 = blockIdx.x * kRows;
  const BatchInfo bi = resolve_batch(P, b);
  const int g = h / P.group;
  const long long qstride = (long long)P.H * D, kstride = (long long)P.Hkv * D;
  const T* qb = q + (bi.q0 * P.H + h) * D;
  const T* kb = k + (bi.k0 * P.Hkv + g) * D;
  const T* vb = v + (bi.k0 * P.Hkv + g) * D;
  const int qvalid = min(kRows, bi.q_len - i0);
  const int rl = warp * 16 + gq, rh = rl + 8;
  const int il = i0 + rl, ih = i0 + rh;
  const float inv_keep = (float)(1.0 / (1.0 - drop_p));
  const unsigned drop_thr = (unsigned)ceil(drop_p * 65536.0);
  float acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float lse_l = INFINITY, lse_h = INFINITY;
  int keys_done = 0;  // weight columns written by pass 2
  if (qvalid > 0) {
    load_rows<T, D>(tq, qb, i0, qvalid, kRows, qstride);
    cp_commit();
    long long jend = bi.kv_len;
    if (P.causal != SDPA_CAUSAL_NONE) jend = min(jend, (long long)bi.offset + i0 + qvalid);
    const int nkt = jend > 0 ? (int)((jend + kKeys - 1) / kKeys) : 0;

    // pass 1: row log-sum-exp (log2 units)
    float m_l = -INFINITY, m_h = -INFINITY, l_l = 0.f, l_h = 0.f;
    if (nkt > 0) {
      load_rows<T, D>(tk[0], kb, 0, min(kKeys, P.Lk), kKeys, kstride);
      cp_commit();
    }
    for (int t = 0; t < nkt; ++t) {
      if (t + 1 < nkt) {
        load_rows<T, D>(tk[(t + 1) & 1], kb, (long long)(t + 1) * kKeys, min(kKeys, P.Lk - (t + 1) * kKeys), kKeys,
                        kstride);
        cp_commit();
        cp_wait<1>();
      } else {
        cp_wait<0>();
      }
      __syncthreads();
      float s[kKeys / 8][4];
#pragma unroll
      for (int n = 0; n < kKeys / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        frag_a(tq, warp * 16, kk * 16, a);
#pragma unroll
        for (int np = 0; np < kKeys / 16; ++np) {
          uint32_t bb[4];
          frag_b_nk(tk[t & 1], np * 16, kk * 16, bb);
          mma<T>(s[2 * np], a, bb[0], bb[1]);
          mma<T>(s[2 * np + 1], a, bb[2], bb[3]);
        }
      }
#pragma unroll
      for (int n = 0; n < kKeys / 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = t * kKeys + n * 8 + 2 * tq4 + (e & 1);
          const int i = (e < 2) ? il : ih;
          if (!(i < bi.q_len && allowed(P, bi, b, h, i, j))) continue;
          const float x = logit2(P, b, h, i, j, s[n][e]);
          float& m = (e < 2) ? m_l : m_h;
          float& l = (e < 2) ? l_l : l_h;
          if (x > m) {
            l = l * exp2f(m - x) + 1.f;
            m = x;
          } else {
            l += exp2f(x - m);
          }
        }
      }
      __syncthreads();
    }
    {
      const float M_l = quad_max(m_l), M_h = quad_max(m_h);
      const float sl = quad_sum(m_l == -INFINITY ? 0.f : l_l * exp2f(m_l - M_l));
      const float sh = quad_sum(m_h == -INFINITY ? 0.f : l_h * exp2f(m_h - M_h));
      lse_l = sl > 0.f ? M_l + log2f(sl) : INFINITY;
      lse_h = sh > 0.f ? M_h + log2f(sh) : INFINITY;
    }

    // pass 2: weights (stored) and out += w' V
    if (nkt > 0) {
      load_rows<T, D>(tk[0], kb, 0, min(kKeys, P.Lk), kKeys, kstride);
      load_rows<T, D>(tv[0], vb, 0, min(kKeys, P.Lk), kKeys, kstride);
      cp_commit();
    }
    for (int t = 0; t < nkt; ++t) {
      if (t + 1 < nkt) {
        const long long r0 = (long long)(t + 1) * kKeys;
        const int valid = min(kKeys, P.Lk - (t + 1) * kKeys);
        load_rows<T, D>(tk[(t + 1) & 1], kb, r0, valid, kKeys, kstride);
        load_rows<T, D>(tv[(t + 1) & 1], vb, r0, valid, kKeys, kstride);
        cp_commit();
        cp_wait<1>();
      } else {
        cp_wait<0>();
      }
      __syncthreads();
      float s[kKeys / 8][4];
#pragma unroll
      for (int n = 0; n < kKeys / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        frag_a(tq, warp * 16, kk * 16, a);
#pragma unroll
        for (int np = 0; np < kKeys / 16; ++np) {
          uint32_t bb[4];
          frag_b_nk(tk[t & 1], np * 16, kk * 16, bb);
          mma<T>(s[2 * np], a, bb[0], bb[1]);
          mma<T>(s[2 * np + 1], a, bb[2], bb[3]);
        }
      }
#pragma unroll
      for (int n = 0; n < kKeys / 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = t * kKeys + n * 8 + 2 * tq4 + (e & 1);
          const int i = (e < 2) ? il : ih;
          const float L = (e < 2) ? lse_l : lse_h;
          float w = 0.f;
          if (i < bi.q_len && allowed(P, bi, b, h, i, j)) {
            w = exp2f(logit2(P, b, h, i, j, s[n][e]) - L);
            if (drop_p > 0.0) {
              const unsigned long long idx = (((unsigned long long)b * P.H + h) * P.Lq + i) * P.Lk + j;
              w = keep(seed, idx, drop_thr) ? w * inv_keep : 0.f;
            }
          }
          s[n][e] = w;
          if (i < P.Lq && j < P.Lk) {
            const T val = (i < bi.q_len && L == INFINITY) ? nan_of<T>() : from_f32<T>(w);
            weights[(((long long)b * P.H + h) * P.Lq + i) * P.Lk + j] = val;
          }
        }
      }
#pragma unroll
      for (int ks = 0; ks < kKeys / 16; ++ks) {
        const uint32_t a[4] = {pk<T>(s[2 * ks][0], s[2 * ks][1]), pk<T>(s[2 * ks][2], s[2 * ks][3]),
                               pk<T>(s[2 * ks + 1][0], s[2 * ks + 1][1]), pk<T>(s[2 * ks + 1][2], s[2 * ks + 1][3])};
#pragma unroll
        for (int nd = 0; nd < D / 16; ++nd) {
          uint32_t bb[4];
          frag_b_kn(tv[t & 1], ks * 16, nd * 16, bb);
          mma<T>(acc[2 * nd], a, bb[0], bb[1]);
          mma<T>(acc[2 * nd + 1], a, bb[2], bb[3]);
        }
      }
      __syncthreads();
    }
    keys_done = nkt * kKeys;
    cp_wait<0>();
    __syncthreads();
  }
  // the weight columns pass 2 did not reach: 0, or NaN for a row with no attended key
  for (int rr = 0; rr < 16; ++rr) {
    const int r = warp * 16 + rr, i = i0 + r;
    if (i >= P.Lq) break;
    const bool nan_row = i < bi.q_len && __shfl_sync(0xffffffffu, (rr < 8) ? lse_l : lse_h, (rr % 8) * 4) == INFINITY;
    T* wrow = weights + (((long long)b * P.H + h) * P.Lq + i) * P.Lk;
    const T fill = nan_row ? nan_of<T>() : from_f32<T>(0.f);
    for (int j = keys_done + lane; j < P.Lk; j += 32) wrow[j] = fill;
  }
  // out: NaN for a row with no attended key, 0 past q_lengths
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = half ? rh : rl, i = i0 + r;
    if (i >= P.Lq) continue;
    const float L = half ? lse_h : lse_l;
    const bool pad = i >= bi.q_len, nan_row = !pad && L == INFINITY;
    T* dst = out + ((bi.q0 + i) * P.H + h) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const float x0 = pad ? 0.f : (nan_row ? __int_as_float(0x7fc00000) : acc[n][2 * half]);
      const float x1 = pad ? 0.f : (nan_row ? __int_as_float(0x7fc00000) : acc[n][2 * half + 1]);
      *reinterpret_cast<uint32_t*>(dst + n * 8 + 2 * tq4) = pk<T>(x0, x1);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
weights_simt_kernel(Problem P, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                    T* __restrict__ out, T* __restrict__ weights, double drop_p, unsigned long long seed) {
  extern __shared__ float qsm[];  // [kWarps][D]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long row = (long long)blockIdx.x * kWarps + warp;  // (b, i, h), h fastest
  if (row >= (long long)P.B * P.Lq * P.H) return;
  const int h = (int)(row % P.H), i = (int)((row / P.H) % P.Lq), b = (int)(row / ((long long)P.H * P.Lq));
  const BatchInfo bi = resolve_batch(P, b);
  const int D = P.D, Dv = P.Dv, g = h / P.group;
  const long long qi = (bi.q0 + i) * P.H + h;
  T* wrow = weights + (((long long)b * P.H + h) * P.Lq + i) * P.Lk;
  T* orow = out + qi * Dv;
  if (i >= bi.q_len) {
    for (int j = lane; j < P.Lk; j += 32) wrow[j] = from_f32<T>(0.f);
    for (int e = lane; e < Dv; e += 32) orow[e] = from_f32<T>(0.f);
    return;
  }
  float* qs = qsm + warp * D;
  for (int c = lane; c < D; c += 32) qs[c] = to_f32(q[qi * D + c]);
  __syncwarp();
  auto logit = [&](int j) -> float {  // log2 units, -inf where not attended
    if (!allowed(P, bi, b, h, i, j)) return -INFINITY;
    const T* kr = k + ((bi.k0 + j) * P.Hkv + g) * D;
    float dot = 0.f;
    for (int c = 0; c < D; ++c) dot = fmaf(qs[c], to_f32(kr[c]), dot);
    return logit2(P, b, h, i, j, dot);
  };
  float m = -INFINITY, l = 0.f;
  for (int j0 = 0; j0 < P.Lk; j0 += 32) {
    const int j = j0 + lane;
    const float x = j < P.Lk ? logit(j) : -INFINITY;
    float mx = x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float m_new = fmaxf(m, mx);
    if (m_new == -INFINITY) continue;
    float p = x == -INFINITY ? 0.f : exp2f(x - m_new);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
    l = l * (m == -INFINITY ? 0.f : exp2f(m - m_new)) + p;
    m = m_new;
  }
  if (!(l > 0.f)) {  // no attended key
    for (int j = lane; j < P.Lk; j += 32) wrow[j] = nan_of<T>();
    for (int e = lane; e < Dv; e += 32) orow[e] = nan_of<T>();
    return;
  }
  const float L = m + log2f(l), inv_keep = (float)(1.0 / (1.0 - drop_p));
  const unsigned drop_thr = (unsigned)ceil(drop_p * 65536.0);
  float o[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) o[u] = 0.f;
  for (int j0 = 0; j0 < P.Lk; j0 += 32) {
    const int j = j0 + lane;
    float w = 0.f;
    if (j < P.Lk) {
      const float x = logit(j);
      if (x != -INFINITY) {
        w = exp2f(x - L);
        if (drop_p > 0.0) {
          const unsigned long long idx = (((unsigned long long)b * P.H + h) * P.Lq + i) * P.Lk + j;
          w = keep(seed, idx, drop_thr) ? w * inv_keep : 0.f;
        }
      }
      wrow[j] = from_f32<T>(w);
    }
    const int n = min(32, P.Lk - j0);
    for (int t = 0; t < n; ++t) {
      const float wt = __shfl_sync(0xffffffffu, w, t);
      if (wt == 0.f) continue;  // warp-uniform
      const T* vr = v + ((bi.k0 + j0 + t) * P.Hkv + g) * Dv;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = lane + 32 * u;
        if (e < Dv) o[u] = fmaf(wt, to_f32(vr[e]), o[u]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int e = lane + 32 * u;
    if (e < Dv) orow[e] = from_f32<T>(o[u]);
  }
}

template <typename T, int D>
cudaError_t launch_mma(const Problem& P, const void* q, const void* k, const void* v, void* out, void* weights,
                       double drop_p, unsigned long long seed, cudaStream_t stream) {
  const size_t smem = (size_t)5 * kRows * D * 2;
  cudaError_t e = cudaFuncSetAttribute(weights_mma_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((P.Lq + kRows - 1) / kRows), (unsigned)P.H, (unsigned)P.B);
  weights_mma_kernel<T, D><<<grid, kWarps * 32, smem, stream>>>(P, (const T*)q, (const T*)k, (const T*)v, (T*)out,
                                                                (T*)weights, drop_p, seed);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_simt(const Problem& P, const void* q, const void* k, const void* v, void* out, void* weights,
                        double drop_p, unsigned long long seed, cudaStream_t stream) {
  const long long rows = (long long)P.B * P.Lq * P.H;
  const dim3 grid((unsigned)((rows + kWarps - 1) / kWarps));
  weights_simt_kernel<T><<<grid, kWarps * 32, sizeof(float) * kWarps * P.D, stream>>>(
      P, (const T*)q, (const T*)k, (const T*)v, (T*)out, (T*)weights, drop_p, seed);
  return cudaGetLastError();
}

}  // namespace

bool weights_mma_supported(const Problem& P, const void* q, const void* k, const void* v, const void* out) {
  if (P.dtype != SDPA_BF16 && P.dtype != SDPA_F16) return false;
  if (P.D != P.Dv || (P.D != 64 && P.D != 128)) return false;
  if (P.q_start || P.H > 65535 || P.B > 65535) return false;
  for (const void* p : {q, k, v, out})
    if (reinterpret_cast<uintptr_t>(p) % 16) return false;
  return true;
}

cudaError_t launch_weights(const Problem& P, bool tiles, const void* q, const void* k, const void* v, void* out,
                           void* weights, double drop_p, unsigned long long seed, cudaStream_t stream) {
  if ((long long)P.B * P.Lq * P.H == 0) return cudaSuccess;
  if (tiles) {
    if (P.dtype == SDPA_BF16)
      return P.D == 128 ? launch_mma<__nv_bfloat16, 128>(P, q, k, v, out, weights, drop_p, seed, stream)
                        : launch_mma<__nv_bfloat16, 64>(P, q, k, v, out, weights, drop_p, seed, stream);
    return P.D == 128 ? launch_mma<__half, 128>(P, q, k, v, out, weights, drop_p, seed, stream)
                      : launch_mma<__half, 64>(P, q, k, v, out, weights, drop_p, seed, stream);
  }
  switch (P.dtype) {
    case SDPA_F32: return launch_simt<float>(P, q, k, v, out, weights, drop_p, seed, stream);
    case SDPA_F16: return launch_simt<__half>(P, q, k, v, out, weights, drop_p, seed, stream);
    default: return launch_simt<__nv_bfloat16>(P, q, k, v, out, weights, drop_p, seed, stream);
  }
}

}  // namespace sdpa
