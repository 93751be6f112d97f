// Rotary position embedding of query / key rows, the step the Keras thread "MultiHeadAttention
// is missing a position_bias call argument" places after the projections (rotary embeddings
// applied to the key and query). The form used: the pair (c, c + d/2) of row t is rotated by
// the angle positions[t] * base^(-2c/d).
//
// An HBM-bound elementwise pass: one thread per pair, consecutive threads on consecutive c of a
// row, so both halves are read and written in coalesced runs. The angle, its sine and cosine
// and the rotation are taken in double precision, so fp32 rows keep full accuracy at positions
// of 10^5 and more. Each pair is read before it is written by the same thread, so out may
// alias x.
#include "device_common.cuh"

namespace sdpa {
namespace {

template <typename T>
__global__ void __launch_bounds__(256)
rope_kernel(const T* x, T* out, long long rows, int nheads, int d, const int32_t* __restrict__ positions,
            double log2_base) {
  const int half = d / 2;
  const long long pairs = rows * nheads * half;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < pairs;
       idx += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(idx % half);
    const long long rh = idx / half;  // (row, head)
    const long long t = rh / nheads;
    const double a = (double)positions[t] * exp2(-2.0 * (double)c / (double)d * log2_base);
    double sn, cs;
    sincos(a, &sn, &cs);
    const double x0 = to_f32(x[rh * d + c]), x1 = to_f32(x[rh * d + c + half]);
    out[rh * d + c] = from_f32<T>((float)(x0 * cs - x1 * sn));
    out[rh * d + c + half] = from_f32<T>((float)(x1 * cs + x0 * sn));
  }
}

template <typename T>
cudaError_t launch_t(const void* x, void* out, long long rows, int nheads, int d, const int32_t* positions,
                     double base, cudaStream_t stream) {
  const long long pairs = rows * nheads * (d / 2);
  if (pairs == 0) return cudaSuccess;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long blocks = (pairs + 255) / 256;
  const unsigned grid = (unsigned)(blocks < 16LL * sms ? blocks : 16LL * sms);
  rope_kernel<T><<<grid, 256, 0, stream>>>((const T*)x, (T*)out, rows, nheads, d, positions, log2(base));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rope(int dtype, const void* x, void* out, long long rows, int nheads, int d,
                        const int32_t* positions, double base, cudaStream_t stream) {
  switch (dtype) {
    case SDPA_F32: return launch_t<float>(x, out, rows, nheads, d, positions, base, stream);
    case SDPA_F16: return launch_t<__half>(x, out, rows, nheads, d, positions, base, stream);
    default: return launch_t<__nv_bfloat16>(x, out, rows, nheads, d, positions, base, stream);
  }
}

}  // namespace sdpa
