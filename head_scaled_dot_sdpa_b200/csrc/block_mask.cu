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
// Two passes. The first streams the uint8 mask once (HBM-bound): each CTA takes a run of 8
// blocks of one block row, so that the grid has many equal CTAs, and loads the next block
// while it reduces the current one; each thread turns 32 mask bytes into one word with a
// SIMD-within-a-register test of non-zero bytes, the CTA sums the set bits, and writes the
// class (and the bits of a PARTIAL block). The second pass builds each block row's ordered list from the classes with one
// warp per row (ballot compaction): the result does not depend on the order in which blocks
// were classified.
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

// Loads of the words of one block that this thread owns (WPT words of 32 mask bytes).
template <int WPT>
struct BlockBytes {
  uint4 a[WPT], b[WPT];
};

template <int WPT, bool kVec>
__device__ __forceinline__ void load_block(BlockBytes<WPT>& x, const uint8_t* base, long long ms_q,
                                           int words, int words_per_row, int rows_valid, int cols_valid) {
#pragma unroll
  for (int u = 0; u < WPT; ++u) {
    const int w = threadIdx.x + u * kThreads;
    x.a[u] = x.b[u] = make_uint4(0, 0, 0, 0);
    if (kVec && w < words) {
      const int r = w / words_per_row, c0 = (w % words_per_row) * 32;
      if (r < rows_valid && c0 + 32 <= cols_valid) {
        const uint4* src = reinterpret_cast<const uint4*>(base + (long long)r * ms_q + c0);
        x.a[u] = __ldcs(src);
        x.b[u] = __ldcs(src + 1);
      }
    }
  }
}

// grid (ceil(nkb / kBlocksPerCta), nqb, H): each CTA classifies kBlocksPerCta consecutive
// blocks of one block row, loading block kb+1 while it reduces block kb.
constexpr int kBlocksPerCta = 8;

template <int WPT, bool kVec>
__global__ void __launch_bounds__(kThreads)
block_classify_kernel(const uint8_t* __restrict__ mask, long long ms_q, long long ms_h, int Lq,
                      int Lk, int bq, int bk, int nqb, int nkb, uint8_t* __restrict__ cls,
                      uint32_t* __restrict__ bits) {
  __shared__ int red[2][kThreads / 32];
  const int qb = blockIdx.y, h = blockIdx.z;
  const int kb0 = blockIdx.x * kBlocksPerCta, kb1 = min(nkb, kb0 + kBlocksPerCta);
  const int words_per_row = bk / 32;
  const int words = bq * words_per_row;
  const int rows_valid = min(bq, Lq - qb * bq);
  const uint8_t* row0 = mask + (long long)h * ms_h + (long long)qb * bq * ms_q;
  BlockBytes<WPT> b0, b1;
  // block kb from `cur` (loaded), the next block's loads into `nxt`; red[] is double-buffered
  // by block parity, so one barrier per block suffices
  auto process = [&](int kb, BlockBytes<WPT>& cur, BlockBytes<WPT>& nxt, int par) {
    if (kb + 1 < kb1)
      load_block<WPT, kVec>(nxt, row0 + (long long)(kb + 1) * bk, ms_q, words, words_per_row, rows_valid,
                            min(bk, Lk - (kb + 1) * bk));
    const int cols_valid = min(bk, Lk - kb * bk);
    const uint8_t* base = row0 + (long long)kb * bk;
    uint32_t w_reg[WPT];
    int local = 0;
#pragma unroll
    for (int u = 0; u < WPT; ++u) {
      const int w = threadIdx.x + u * kThreads;
      uint32_t word = 0;
      if (w < words) {
        const int r = w / words_per_row, c0 = (w % words_per_row) * 32;
        if (r < rows_valid && c0 < cols_valid) {
          if (kVec && c0 + 32 <= cols_valid) {
            word = word_from_16(cur.a[u], cur.b[u]);
          } else {
            const uint8_t* src = base + (long long)r * ms_q + c0;
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
    if ((threadIdx.x & 31) == 0) red[par][threadIdx.x / 32] = local;
    __syncthreads();
    int set = 0;
#pragma unroll
    for (int x = 0; x < kThreads / 32; ++x) set += red[par][x];
    const int cells = rows_valid * cols_valid;
    const uint8_t c = set == 0 ? SDPA_BLOCK_EMPTY : (set == cells ? SDPA_BLOCK_FULL : SDPA_BLOCK_PARTIAL);
    const long long blk = ((long long)h * nqb + qb) * nkb + kb;
    if (c == SDPA_BLOCK_PARTIAL) {
      uint32_t* dst = bits + blk * words;
#pragma unroll
      for (int u = 0; u < WPT; ++u) {
        const int w = threadIdx.x + u * kThreads;
        if (w < words) dst[w] = w_reg[u];
      }
    }
    if (threadIdx.x == 0) cls[blk] = c;
  };
  load_block<WPT, kVec>(b0, row0 + (long long)kb0 * bk, ms_q, words, words_per_row, rows_valid,
                        min(bk, Lk - kb0 * bk));
  for (int kb = kb0; kb < kb1; kb += 2) {
    process(kb, b0, b1, 0);
    if (kb + 1 < kb1) process(kb + 1, b1, b0, 1);
  }
}

// One warp per block row: the non-empty blocks in increasing kb, as kb | class << 30.
__global__ void __launch_bounds__(kThreads)
block_list_kernel(const uint8_t* __restrict__ cls, int rows, int nkb, int32_t* __restrict__ count,
                  uint32_t* __restrict__ list) {
  const int row = blockIdx.x * (kThreads / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const uint8_t* c_row = cls + (long long)row * nkb;
  uint32_t* l_row = list + (long long)row * nkb;
  int n = 0;
  for (int kb0 = 0; kb0 < nkb; kb0 += 32) {
    const int kb = kb0 + lane;
    const uint32_t c = kb < nkb ? c_row[kb] : (uint32_t)SDPA_BLOCK_EMPTY;
    const bool ne = c != SDPA_BLOCK_EMPTY;
    const uint32_t ball = __ballot_sync(0xffffffffu, ne);
    if (ne) l_row[n + __popc(ball & ((1u << lane) - 1u))] = (uint32_t)kb | (c << 30);
    n += __popc(ball);
  }
  if (lane == 0) count[row] = n;
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
  const dim3 grid((unsigned)((nkb + kBlocksPerCta - 1) / kBlocksPerCta), (unsigned)nqb, (unsigned)H);
  const bool small = bq * bk <= 2 * 32 * kThreads;  // at most 2 words of 32 bytes per thread
#define SDPA_CLASSIFY(WPT, VEC)                                                                   \
  block_classify_kernel<WPT, VEC><<<grid, kThreads, 0, stream>>>(mask, ms[1], ms[2], Lq, Lk, bq, bk, \
                                                                 nqb, nkb, cls, bits)
  if (small) {
    if (vec) SDPA_CLASSIFY(2, true); else SDPA_CLASSIFY(2, false);
  } else {
    if (vec) SDPA_CLASSIFY(kMaxWordsPerThread, true); else SDPA_CLASSIFY(kMaxWordsPerThread, false);
  }
#undef SDPA_CLASSIFY
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int rows = H * nqb;
  const int per = kThreads / 32;
  block_list_kernel<<<(rows + per - 1) / per, kThreads, 0, stream>>>(cls, rows, nkb, count, list);
  return cudaGetLastError();
}

}  // namespace sdpa
