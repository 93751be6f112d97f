// Building blocks of the mma.sync tile kernels (the fused gradient and the materialized
// weights): cp.async staging of 16-bit row tiles into XOR-swizzled shared memory, ldmatrix
// fragment loads, m16n8k16 MMAs with fp32 accumulation, and the masking test of
// NNlib.scaled_dot_product_attention (Flux.jl page "Neural Network primitives from NNlib.jl":
// kv_lengths, is_causal with q_offset, mask).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device_common.cuh"

namespace sdpa {
namespace tiles {

constexpr int kWarps = 4;  // every tile kernel runs 4 warps
constexpr float kLog2e = 1.4426950408889634f;

template <typename T> struct IsBf16;
template <> struct IsBf16<__nv_bfloat16> { static constexpr bool value = true; };
template <> struct IsBf16<__half> { static constexpr bool value = false; };

__device__ __forceinline__ uint32_t su32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N> __device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

template <typename T>
__device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (IsBf16<T>::value) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

template <typename T> __device__ __forceinline__ uint32_t pk(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pk<__nv_bfloat16>(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <> __device__ __forceinline__ uint32_t pk<__half>(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// x0, x1 as the sum of two 16-bit pairs, hi = round(x) and lo = round(x - hi): the products of
// an MMA on hi and on lo add up to the fp32 operand's product to about 2^-16 relative, where one
// rounding alone would leave 2^-9 (bf16) in every weight and dx of the gradient's sums.
template <typename T>
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pk<T>(x0, x1);
  float h0, h1;
  if constexpr (IsBf16<T>::value) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&hi);
    h0 = __low2float(v);
    h1 = __high2float(v);
  } else {
    const __half2 v = *reinterpret_cast<const __half2*>(&hi);
    h0 = __low2float(v);
    h1 = __high2float(v);
  }
  lo = pk<T>(x0 - h0, x1 - h1);
}

// A tile of `rows` x D 16-bit elements in shared memory: row r, 16-byte chunk c lives at chunk
// slot r * (D/8) + (c ^ (r & 7)), so the 8 rows an ldmatrix reads hit 8 different bank groups.
template <int D>
struct Tile {
  static constexpr int kC = D / 8;
  uint32_t base;
  __device__ __forceinline__ uint32_t at(int r, int col) const {
    return base + (uint32_t)((r * kC + ((col >> 3) ^ (r & 7))) * 16);
  }
};

// Rows [row0, row0 + rows) of a (rows, heads, D) array at head h into a tile; rows at or past
// `valid` are zero-filled (no global read). All threads of the CTA take part.
template <typename T, int D>
__device__ __forceinline__ void load_rows(const Tile<D>& t, const T* g, long long row0, int valid, int rows,
                                          long long row_stride) {
  constexpr int kC = D / 8;
  for (int idx = threadIdx.x; idx < rows * kC; idx += kWarps * 32) {
    const int r = idx / kC, c = idx % kC;
    const bool ok = r < valid;
    const T* src = ok ? g + (row0 + r) * row_stride + c * 8 : g;
    cp16(t.base + (uint32_t)((r * kC + (c ^ (r & 7))) * 16), src, ok ? 16 : 0);
  }
}

// A operand (16 x 16, row-major) from rows r0.., columns k0.. of a tile.
template <int D>
__device__ __forceinline__ void frag_a(const Tile<D>& t, int r0, int k0, uint32_t (&a)[4]) {
  const int lane = threadIdx.x % 32;
  ldsm4(t.at(r0 + (lane % 8) + 8 * ((lane / 8) % 2), k0 + 8 * (lane / 16)), a);
}
// B operands of two 8-wide n tiles (n0.., n0+8..) at k0.. from a tile stored [n][k]
// (b[0], b[1]: first n tile; b[2], b[3]: second).
template <int D>
__device__ __forceinline__ void frag_b_nk(const Tile<D>& t, int n0, int k0, uint32_t (&b)[4]) {
  const int lane = threadIdx.x % 32;
  ldsm4(t.at(n0 + (lane % 8) + 8 * (lane / 16), k0 + 8 * ((lane / 8) % 2)), b);
}
// The same from a tile stored [k][n] (transposing ldmatrix).
template <int D>
__device__ __forceinline__ void frag_b_kn(const Tile<D>& t, int k0, int n0, uint32_t (&b)[4]) {
  const int lane = threadIdx.x % 32;
  ldsm4t(t.at(k0 + (lane % 8) + 8 * ((lane / 8) % 2), n0 + 8 * (lane / 16)), b);
}

__device__ __forceinline__ float quad_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

// Whether query i (< q_len) may attend key j.
__device__ __forceinline__ bool allowed(const Problem& P, const BatchInfo& bi, int b, int h, int i, int j) {
  if (j >= bi.kv_len) return false;
  if (P.causal != SDPA_CAUSAL_NONE && (long long)j > (long long)bi.offset + i) return false;
  return mask_allows(P, b, h, i, j);
}

}  // namespace tiles
}  // namespace sdpa
