// Rotary position embedding of query / key rows, the step the Keras thread "MultiHeadAttention
// is missing a position_bias call argument" places after the projections (rotary embeddings
// applied to the key and query). The form used: the pair (c, c + d/2) of row t is rotated by
// the angle positions[t] * base^(-2c/d).
//
// An HBM-bound elementwise pass. The angle of (row t, pair c) is the same for every head, so one
// thread takes VEC consecutive pairs of one row, computes their sines and cosines once and
// rotates those pairs in several heads; the threads of a warp cover consecutive pairs, so each
// head's two halves are read and written in coalesced runs. With 16-bit data (VEC = 8: 16-byte
// runs) a thread takes up to 8 heads and issues all 16 loads before the first is used.
// The frequencies base^(-2c/d) are a per-block table in double precision. The angle is formed
// and reduced to [-pi, pi] in double precision (positions of 10^5 and more keep their accuracy:
// a - 2 pi * rint(a / (2 pi)), the quotient taken as a product with 1 / (2 pi)), then CUDA's
// single-precision sine and cosine evaluate it: sincosf for fp32 data, the __sincosf intrinsic
// (absolute error about 2^-21 on [-pi, pi], far below the 16-bit types' resolution) for bf16 /
// fp16 data. Each element is read before it is written by the same thread, so out may alias x.
#include "device_common.cuh"

namespace sdpa {
namespace {

constexpr int kThreads = 256;
// the 16-byte path: small blocks spread its items (8 pairs of one row in up to 8 heads) evenly
// over the SMs
constexpr int kThreadsVec8 = 128;
constexpr double kTwoPi = 6.283185307179586476925286766559;
constexpr double kInvTwoPi = 0.15915494309189533576888376337251;

// (sin, cos) of the angle a (radians, any size), reduced to [-pi, pi] in double precision
template <bool kFast>
__device__ __forceinline__ void angle_sincos(double a, float* sn, float* cs) {
  const double r = fma(-rint(a * kInvTwoPi), kTwoPi, a);
  if constexpr (kFast)
    __sincosf((float)r, sn, cs);
  else
    sincosf((float)r, sn, cs);
}

template <typename T, int VEC>
__global__ void __launch_bounds__(kThreads)
rope_kernel(const T* x, T* out, long long rows, int nheads, int d, const int32_t* __restrict__ positions,
            double log2_base) {
  extern __shared__ double freq[];  // [d / 2]
  const int half = d / 2;
  const int groups = half / VEC;  // pair groups per row
  const long long row_elems = (long long)nheads * d;
  auto fill_table = [&]() {
    for (int c = threadIdx.x; c < half; c += blockDim.x) freq[c] = exp2(-2.0 * (double)c / (double)d * log2_base);
    __syncthreads();
  };
  if constexpr (VEC == 8 && sizeof(T) == 2) {
    // item = (row, 8 pairs, up to kHeads heads): consecutive threads take consecutive 16-byte
    // runs of one head's halves; all of an item's loads are issued before the first is used,
    // the first item's before the block builds its frequency table
    constexpr int kHeads = 8;
    const int nhc = (nheads + kHeads - 1) / kHeads;
    const long long items = rows * groups * nhc;
    const long long stride = (long long)gridDim.x * blockDim.x;
    long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    uint4 a[kHeads], b[kHeads];
    int c0 = 0, h0 = 0;
    long long t = 0;
    auto load = [&]() {
      c0 = (int)(idx % groups) * VEC;
      const long long rest = idx / groups;
      h0 = (int)(rest % nhc) * kHeads;
      t = rest / nhc;
      const T* xr = x + t * row_elems + (long long)h0 * d + c0;
#pragma unroll
      for (int g = 0; g < kHeads; ++g) {
        if (h0 + g < nheads) {
          a[g] = *reinterpret_cast<const uint4*>(xr + (long long)g * d);
          b[g] = *reinterpret_cast<const uint4*>(xr + (long long)g * d + half);
        }
      }
    };
    if (idx < items) load();
    fill_table();
    for (; idx < items;) {
      const double pos = (double)positions[t];
      float cs[VEC], sn[VEC];
#pragma unroll
      for (int u = 0; u < VEC; ++u) angle_sincos<true>(pos * freq[c0 + u], &sn[u], &cs[u]);
      T* orow = out + t * row_elems + (long long)h0 * d + c0;
#pragma unroll
      for (int g = 0; g < kHeads; ++g) {
        if (h0 + g >= nheads) break;
        const T* pa = reinterpret_cast<const T*>(&a[g]);
        const T* pb = reinterpret_cast<const T*>(&b[g]);
        uint4 ya, yb;
        T* qa = reinterpret_cast<T*>(&ya);
        T* qb = reinterpret_cast<T*>(&yb);
#pragma unroll
        for (int u = 0; u < VEC; ++u) {
          const float x0 = to_f32(pa[u]), x1 = to_f32(pb[u]);
          qa[u] = from_f32<T>(x0 * cs[u] - x1 * sn[u]);
          qb[u] = from_f32<T>(x1 * cs[u] + x0 * sn[u]);
        }
        *reinterpret_cast<uint4*>(orow + (long long)g * d) = ya;
        *reinterpret_cast<uint4*>(orow + (long long)g * d + half) = yb;
      }
      idx += stride;
      if (idx < items) load();
    }
  } else {
    // item = (row, pair group) in every head
    fill_table();
    const long long items = rows * groups;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < items;
         idx += (long long)gridDim.x * blockDim.x) {
      const long long t = idx / groups;
      const int c0 = (int)(idx % groups) * VEC;
      const double pos = (double)positions[t];
      float cs[VEC], sn[VEC];
#pragma unroll
      for (int u = 0; u < VEC; ++u) angle_sincos<sizeof(T) == 2>(pos * freq[c0 + u], &sn[u], &cs[u]);
      const T* xr = x + t * row_elems + c0;
      T* orow = out + t * row_elems + c0;
      for (int h = 0; h < nheads; ++h) {
        float x0[VEC], x1[VEC];
#pragma unroll
        for (int u = 0; u < VEC; ++u) {
          x0[u] = to_f32(xr[(long long)h * d + u]);
          x1[u] = to_f32(xr[(long long)h * d + half + u]);
        }
#pragma unroll
        for (int u = 0; u < VEC; ++u) {
          orow[(long long)h * d + u] = from_f32<T>(x0[u] * cs[u] - x1[u] * sn[u]);
          orow[(long long)h * d + half + u] = from_f32<T>(x1[u] * cs[u] + x0[u] * sn[u]);
        }
      }
    }
  }
}

template <typename T>
cudaError_t launch_t(const void* x, void* out, long long rows, int nheads, int d, const int32_t* positions,
                     double base, cudaStream_t stream) {
  const int half = d / 2;
  if (rows == 0 || half == 0) return cudaSuccess;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // 16-bit rows whose halves are whole 16-byte runs (half a multiple of 8, 16-byte aligned
  // arrays): 8 consecutive pairs per thread; otherwise one pair per thread
  const bool vec8 = sizeof(T) == 2 && half % 8 == 0 && (reinterpret_cast<uintptr_t>(x) % 16 == 0) &&
                    (reinterpret_cast<uintptr_t>(out) % 16 == 0);
  const long long items = vec8 ? rows * (half / 8) * ((nheads + 7) / 8) : rows * half;
  const int threads = vec8 ? kThreadsVec8 : kThreads;
  const long long blocks = (items + threads - 1) / threads;
  const long long max_blocks = (vec8 ? 32LL : 8LL) * sms;
  const unsigned grid = (unsigned)(blocks < max_blocks ? blocks : max_blocks);
  const size_t smem = sizeof(double) * half;
  if (vec8)
    rope_kernel<T, 8><<<grid, threads, smem, stream>>>((const T*)x, (T*)out, rows, nheads, d, positions, log2(base));
  else
    rope_kernel<T, 1><<<grid, threads, smem, stream>>>((const T*)x, (T*)out, rows, nheads, d, positions, log2(base));
  return cudaGetLastError();
}

// (cos, sin) of every (row, pair c) angle as an fp16 pair, table[row * (d/2) + c], the angle
// formed and reduced as in rope_kernel. The prefill kernel reads it to rotate its Q tiles in
// shared memory (fp16 keeps 11 significant bits, finer than the bf16 of the rotated values).
__global__ void __launch_bounds__(kThreads)
rope_table_kernel(long long rows, int d, const int32_t* __restrict__ positions, double log2_base,
                  __half2* __restrict__ table) {
  extern __shared__ double freq[];  // [d / 2]
  const int half = d / 2;
  for (int c = threadIdx.x; c < half; c += blockDim.x) freq[c] = exp2(-2.0 * (double)c / (double)d * log2_base);
  __syncthreads();
  const long long items = rows * half;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < items;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long t = idx / half;
    const int c = (int)(idx % half);
    float sn, cs;
    angle_sincos<true>((double)positions[t] * freq[c], &sn, &cs);  // stored as fp16
    table[idx] = __floats2half2_rn(cs, sn);
  }
}

}  // namespace

cudaError_t launch_rope_table(long long rows, int d, const int32_t* positions, double base, void* table,
                              cudaStream_t stream) {
  const int half = d / 2;
  if (rows == 0 || half == 0) return cudaSuccess;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long blocks = (rows * half + kThreads - 1) / kThreads;
  const unsigned grid = (unsigned)(blocks < 8LL * sms ? blocks : 8LL * sms);
  rope_table_kernel<<<grid, kThreads, sizeof(double) * half, stream>>>(rows, d, positions, log2(base),
                                                                       static_cast<__half2*>(table));
  return cudaGetLastError();
}

cudaError_t launch_rope(int dtype, const void* x, void* out, long long rows, int nheads, int d,
                        const int32_t* positions, double base, cudaStream_t stream) {
  switch (dtype) {
    case SDPA_F32: return launch_t<float>(x, out, rows, nheads, d, positions, base, stream);
    case SDPA_F16: return launch_t<__half>(x, out, rows, nheads, d, positions, base, stream);
    default: return launch_t<__nv_bfloat16>(x, out, rows, nheads, d, positions, base, stream);
  }
}

}  // namespace sdpa
