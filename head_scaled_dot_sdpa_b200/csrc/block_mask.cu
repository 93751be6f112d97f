// Block classification of a dynamic boolean mask, after the splash-attention mask info of the
// JAX pull request "Support dynamic masks in splash attention" (block_mask with three classes,
// partial_mask_blocks holding the bits of the blocks that are neither empty nor full, and a
// per-step "next block" table). Here, for every block row (head h, query block qb):
//   - each bq x bk block is EMPTY (no attended cell), FULL (every in-range cell attended) or
//     PARTIAL;
//   - the bits of PARTIAL blocks are packed, one 32-bit word per 32 keys of a query row, at
//     the block's own slot (so no counter or compaction is needed, and the result is
//     deterministic);
//   - the non-empty blocks are listed in increasing kb with their class (kb | class << 30),
//     which is what the attention kernel walks, skipping empty blocks outright.
// The kernel streams the uint8 mask once (HBM-bound): one CTA per block row, each thread
// turning 32 mask bytes into one word with a SIMD-within-a-register test of non-zero bytes.
#include "device_common.cuh"

namespace sdpa {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxWordsPerThread = 8;  // bq * bk / 32 <= 2048

// Bits 0..3 = (byte k of x != 0) for k = 0..3.
__device__ __forceinline__ uint32_t nonzero_nibble(uint32_t x) {
  const uint32_t hi = (((x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x) & 0x80808080u;
  return (hi * 0x00204081u) >> 28;
}

__device__ __forceinline__ uint32_t word_from_16(uint4 a, uint4 b) {
  return nonzero_nibble(a.x) | (nonzero_nibble(a.y) << 4) | (nonzero_nibble(a.z) << 8) |
         (nonzero_nibble(a.w) << 12) | (nonzero_nibble(b.x) << 16) | (nonzero_nibble(b.y) << 20) |
         (nonzero_nibble(b.z) << 24) | (nonzero_nibble(b.w) << 28);
}

template <bool kVec>
__global__ void __launch_bounds__(kThreads)
block_classify_kernel(const uint8_t* __restrict__ mask, long long ms_q, long long ms_h, int Lq,
                      int Lk, int bq, int bk, int nqb, int nkb, uint8_t* __restrict__ cls,
                      int32_t* __restrict__ count, uint32_t* __restrict__ list,
                      uint32_t* __restrict__ bits) {
  __shared__ int red[kThreads / 32];
  __shared__ int total;
  const int hq = blockIdx.x;  // h * nqb + qb
  const int h = hq / nqb, qb = hq % nqb;
  const int words_per_row = bk / 32;
  const int words = bq * words_per_row;
  const int rows_valid = min(bq, Lq - qb * bq);
  int n_listed = 0;
  const uint8_t* head = mask + (long long)h * ms_h;

  for (int kb = 0; kb < nkb; ++kb) {
    const int cols_valid = min(bk, Lk - kb * bk);
    uint32_t w_reg[kMaxWordsPerThread];
    int local = 0;
#pragma unroll
    for (int u = 0; u < kMaxWordsPerThread; ++u) {
      const int w = threadIdx.x + u * kThreads;
      uint32_t word = 0;
      if (w < words) {
        const int r = w / words_per_row, wc = w % words_per_row;
        const int c0 = wc * 32;
        if (r < rows_valid && c0 < cols_valid) {
          const uint8_t* src = head + (long long)(qb * bq + r) * ms_q + (long long)kb * bk + c0;
          if (kVec && c0 + 32 <= cols_valid) {
            const uint4 a = __ldcs(reinterpret_cast<const uint4*>(src));
            const uint4 b2 = __ldcs(reinterpret_cast<const uint4*>(src) + 1);
            word = word_from_16(a, b2);
          } else {
            const int n = min(32, cols_valid - c0);
            for (int c = 0; c < n; ++c) word |= (src[c] != 0 ? 1u : 0u) << c;
          }
        }
      }
      w_reg[u] = word;
      local += __popc(word);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = local;
    __syncthreads();
    if (threadIdx.x == 0) {
      int t = 0;
      for (int x = 0; x < kThreads / 32; ++x) t += red[x];
      total = t;
    }
    __syncthreads();
    const int set = total;
    const int cells = rows_valid * cols_valid;
    const uint8_t c = set == 0 ? SDPA_BLOCK_EMPTY : (set == cells ? SDPA_BLOCK_FULL : SDPA_BLOCK_PARTIAL);
    const long long blk = (long long)hq * nkb + kb;
    if (c == SDPA_BLOCK_PARTIAL) {
      uint32_t* dst = bits + blk * words;
#pragma unroll
      for (int u = 0; u < kMaxWordsPerThread; ++u) {
        const int w = threadIdx.x + u * kThreads;
        if (w < words) dst[w] = w_reg[u];
      }
    }
    if (threadIdx.x == 0) {
      cls[blk] = c;
      if (c != SDPA_BLOCK_EMPTY) list[(long long)hq * nkb + (n_listed++)] = (uint32_t)kb | ((uint32_t)c << 30);
    }
    // `total` and `red` are rewritten next iteration only after everyone passed this point.
    __syncthreads();
  }
  if (threadIdx.x == 0) count[hq] = n_listed;
}

}  // namespace

cudaError_t launch_block_classify(const uint8_t* mask, const long long ms[3], int H, int Lq,
                                  int Lk, int bq, int bk, uint8_t* cls, int32_t* count,
                                  uint32_t* list, uint32_t* bits, int* status,
                                  cudaStream_t stream) {
  (void)status;
  const int nqb = (Lq + bq - 1) / bq, nkb = (Lk + bk - 1) / bk;
  const bool vec = (reinterpret_cast<uintptr_t>(mask) % 16 == 0) && (ms[1] % 16 == 0) &&
                   (ms[2] % 16 == 0) && (bk % 32 == 0);
  const dim3 grid((unsigned)(H * nqb));
  if (vec)
    block_classify_kernel<true><<<grid, kThreads, 0, stream>>>(mask, ms[1], ms[2], Lq, Lk, bq, bk,
                                                               nqb, nkb, cls, count, list, bits);
  else
    block_classify_kernel<false><<<grid, kThreads, 0, stream>>>(mask, ms[1], ms[2], Lq, Lk, bq,
                                                                bk, nqb, nkb, cls, count, list, bits);
  return cudaGetLastError();
}

}  // namespace sdpa
