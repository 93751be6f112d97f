// Packed sequences (Flux.jl page "Neural Network primitives from NNlib.jl", entry
// scaled_dot_product_attention, keywords q_segments / kv_segments / maxlen and the paragraph
// "Packed sequences"): the segment lengths live on the device, so the first row of every
// segment is found here, on the device, by one block that scans the lengths in chunks of
// 1024 with a running carry. The attention kernels then read segment b's rows
// [start[b], start[b + 1]) exactly as they read batch element b of a padded batch.
//
// The lengths are checked as they are scanned. A negative length counts as 0. Starts are
// clamped to the array rows, so no kernel reads or writes past the arrays whatever the
// lengths are. A negative length, a length above maxlen, or lengths whose sum differs from
// the array rows set SDPA_ERR_DEVICE_CHECK in the status word. Rows of a segment past maxlen
// are not computed.
#include "device_common.cuh"

namespace sdpa {
namespace {

constexpr int kScanThreads = 1024;

// Exclusive prefix sum over the block of x (>= 0); `total` receives the block's sum.
__device__ long long block_exclusive_scan(long long x, long long* warp_sums, long long& total) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  long long incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    long long w = warp_sums[lane];  // kScanThreads / 32 == 32 warps
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const long long before = warp ? warp_sums[warp - 1] : 0;
  total = warp_sums[31];
  __syncthreads();  // warp_sums is reused by the next call
  return before + incl - x;
}

__global__ void __launch_bounds__(kScanThreads)
segment_starts_kernel(const int32_t* __restrict__ q_segments, const int32_t* __restrict__ kv_segments,
                      int n, int maxlen, int q_total, int kv_total, int32_t* __restrict__ q_start,
                      int32_t* __restrict__ kv_start, int* status) {
  __shared__ long long warp_sums[32];
  long long q_carry = 0, kv_carry = 0;
  bool bad = false;
  for (int c0 = 0; c0 < n; c0 += kScanThreads) {
    const int s = c0 + threadIdx.x;
    long long ql = 0, kl = 0;
    if (s < n) {
      ql = q_segments[s];
      kl = kv_segments[s];
      if (ql < 0 || kl < 0 || ql > maxlen || kl > maxlen) bad = true;
      ql = ql < 0 ? 0 : ql;
      kl = kl < 0 ? 0 : kl;
    }
    long long q_sum, kv_sum;
    const long long qs = q_carry + block_exclusive_scan(ql, warp_sums, q_sum);
    const long long ks = kv_carry + block_exclusive_scan(kl, warp_sums, kv_sum);
    if (s < n) {
      q_start[s] = (int32_t)(qs < q_total ? qs : q_total);
      kv_start[s] = (int32_t)(ks < kv_total ? ks : kv_total);
    }
    q_carry += q_sum;
    kv_carry += kv_sum;
  }
  if (threadIdx.x == 0) {
    q_start[n] = (int32_t)(q_carry < q_total ? q_carry : q_total);
    kv_start[n] = (int32_t)(kv_carry < kv_total ? kv_carry : kv_total);
    if (q_carry != q_total || kv_carry != kv_total) bad = true;
  }
  if (bad) report(status, SDPA_ERR_DEVICE_CHECK);
}

}  // namespace

cudaError_t launch_segment_starts(const int32_t* q_segments, const int32_t* kv_segments, int n,
                                  int maxlen, int q_total, int kv_total, int32_t* q_start,
                                  int32_t* kv_start, int* status, cudaStream_t stream) {
  segment_starts_kernel<<<1, kScanThreads, 0, stream>>>(q_segments, kv_segments, n, maxlen, q_total,
                                                         kv_total, q_start, kv_start, status);
  return cudaGetLastError();
}

}  // namespace sdpa
