// Split-KV attention for decoding with a KV cache (Flux.jl page "Neural Network primitives
// from NNlib.jl", scaled_dot_product_attention: is_causal=:bottom_right and its example
// "decoding with a KV cache"), followed by a cross-split combine.
//
// A decode step reads every valid key/value row of the cache once and does ~4 flops per byte,
// so the kernel is built for HBM streaming:
//  - one CTA per (batch b, key/value head, split of S keys); the grid covers the cache
//    capacity and CTAs past kv_len[b] (known only on the device) exit at once;
//  - the g = nheads/nkvheads query heads that share the key/value head, times the n_new
//    queries, form the (at most 16) rows of one m16 tile, so each K/V byte is read once for
//    all of them;
//  - each of the 4 warps streams its own 16-key tiles through a private 3-stage cp.async ring
//    (16-byte copies, XOR-swizzled rows), so the main loop needs no CTA barrier;
//  - QK^T and PV run on mma.sync m16n8k16 (fp32 accumulate) with the S accumulator reused as
//    the A operand of PV; the online softmax works in the log2 domain (exp2 of
//    scale*log2(e)*s);
//  - the warps' states merge in shared memory, and each CTA writes one partial
//    (unnormalised O, running max, running sum) per row; the combine kernel merges the
//    partials of a row with weights 2^(m_s - M).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device_common.cuh"

namespace sdpa {
namespace {

constexpr int kWarps = 4;
constexpr int kStages = 3;
constexpr int kTileKeys = 16;
constexpr int kRows = 16;

template <typename T> struct MmaName;
template <> struct MmaName<__nv_bfloat16> { static constexpr bool bf16 = true; };
template <> struct MmaName<__half> { static constexpr bool bf16 = false; };

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

template <typename T>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if constexpr (MmaName<T>::bf16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

template <typename T> __device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <> __device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Partial state of one (b, kv head, split, row): O[D] unnormalised, then (m, l) in log2 units.
struct Partials {
  float* o;   // [B][Hkv][max_splits][kRows][D]
  float* ml;  // [B][Hkv][max_splits][kRows][2]
  int max_splits;
  int split;  // keys per split
};

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
decode_split_kernel(Problem P, const T* __restrict__ q, const T* __restrict__ kc,
                    const T* __restrict__ vc, Partials part) {
  constexpr int kChunks = D * 2 / 16;            // 16-byte chunks per row
  constexpr int kTileBytes = kTileKeys * D * 2;  // one K (or V) tile
  constexpr int kDTiles = D / 8;                 // n-tiles of the output
  constexpr int kKSteps = D / 16;                // k-steps of QK^T
  extern __shared__ __align__(128) unsigned char smem[];

  const int s = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_new = P.Lq, cap = P.Lk, gsz = P.group;
  const int idx = P.cache_index[b];
  if (idx < 0 || idx > cap - n_new) return;  // reported by the cache update
  const int kvlen = idx + n_new;
  const int k0 = s * part.split;
  if (k0 >= kvlen) return;
  const int k1 = min(k0 + part.split, kvlen);
  const int R = n_new * gsz;  // rows r = t * gsz + hh
  // range-checked build: keys inside the cache, the split inside the partials, rows in a tile
  if (!SDPA_CHECKED(P.status, k1 <= cap && s < part.max_splits && R <= kRows)) return;
  const int off = kvlen - n_new;  // :bottom_right: query t attends keys j <= off + t

  const int grp = lane / 4, t4 = lane % 4;

  // Q fragments (A operand, rows >= R are zero).
  uint32_t qa[kKSteps][4];
  {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = grp + 8 * half;
      const T* qrow = nullptr;
      if (r < R) {
        const int t = r / gsz, hh = r % gsz;
        qrow = q + (((long long)b * n_new + t) * P.H + (long long)kvh * gsz + hh) * D;
      }
#pragma unroll
      for (int kk = 0; kk < kKSteps; ++kk) {
        uint32_t lo = 0, hi = 0;
        if (qrow) {
          lo = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * t4);
          hi = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 8 + 2 * t4);
        }
        qa[kk][half] = lo;      // a0a1 (row grp) / a2a3 (row grp+8)
        qa[kk][2 + half] = hi;  // a4a5 / a6a7
      }
    }
  }

  unsigned char* ring = smem + warp * kStages * 2 * kTileBytes;
  const uint32_t ring_s = smem_u32(ring);
  const long long row_stride = (long long)P.Hkv * D;  // elements between consecutive keys
  const T* kbase = kc + ((long long)b * cap * P.Hkv + kvh) * D;
  const T* vbase = vc + ((long long)b * cap * P.Hkv + kvh) * D;
  const int n_tiles = (k1 - k0 + kTileKeys - 1) / kTileKeys;
  const int my_tiles = n_tiles > warp ? (n_tiles - warp + kWarps - 1) / kWarps : 0;

  auto issue = [&](int it, int stage) {
    const int key0 = k0 + (warp + it * kWarps) * kTileKeys;
    const uint32_t ks = ring_s + stage * 2 * kTileBytes;
    const uint32_t vs = ks + kTileBytes;
#pragma unroll
    for (int x = lane; x < kTileKeys * kChunks; x += 32) {
      const int r = x / kChunks, c = x % kChunks;
      const int key = key0 + r;
      const bool ok = key < k1;
      const long long goff = (long long)(ok ? key : k0) * row_stride + c * 8;
      const uint32_t so = (uint32_t)(r * kChunks + (c ^ (r & 7))) * 16;
      cp_async16(ks + so, kbase + goff, ok ? 16 : 0);
      cp_async16(vs + so, vbase + goff, ok ? 16 : 0);
    }
  };

#pragma unroll
  for (int st = 0; st < kStages - 1; ++st) {
    if (st < my_tiles) issue(st, st);
    cp_async_commit();
  }

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float oc[kDTiles][4];
#pragma unroll
  for (int d = 0; d < kDTiles; ++d) oc[d][0] = oc[d][1] = oc[d][2] = oc[d][3] = 0.f;

  for (int it = 0; it < my_tiles; ++it) {
    if (it + kStages - 1 < my_tiles) issue(it + kStages - 1, (it + kStages - 1) % kStages);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const uint32_t ks = ring_s + (it % kStages) * 2 * kTileBytes;
    const uint32_t vs = ks + kTileBytes;
    const int key0 = k0 + (warp + it * kWarps) * kTileKeys;

    // S = Q K^T over the tile's 16 keys (two n8 tiles).
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < kKSteps; ++kk) {
      const int mtx = lane / 8, rr = lane % 8;
      const int key = ((mtx >> 1) << 3) + rr;
      const int chunk = 2 * kk + (mtx & 1);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(ks + (uint32_t)(key * kChunks + (chunk ^ (key & 7))) * 16, b0, b1, b2, b3);
      mma16816<T>(sc[0], qa[kk], b0, b1);
      mma16816<T>(sc[1], qa[kk], b2, b3);
    }

    // Mask (split end / kv length, and :bottom_right causality), then online softmax.
    float x[2][4];
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int half = e >> 1;
        const int r = grp + 8 * half;
        const int key = key0 + nt * 8 + 2 * t4 + (e & 1);
        const int t = r / gsz;
        const bool ok = key < k1 && key <= off + t;
        x[nt][e] = ok ? sc[nt][e] * P.scale_log2 : -INFINITY;
        mx[half] = fmaxf(mx[half], x[nt][e]);
      }
    float alpha[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      mx[half] = fmaxf(mx[half], __shfl_xor_sync(0xffffffffu, mx[half], 1));
      mx[half] = fmaxf(mx[half], __shfl_xor_sync(0xffffffffu, mx[half], 2));
      const float m_new = fmaxf(m_run[half], mx[half]);
      alpha[half] = (m_new == -INFINITY) ? 1.f : exp2f(m_run[half] - m_new);
      m_run[half] = m_new;
    }
    float ps[2][4];
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int half = e >> 1;
        const float p = (x[nt][e] == -INFINITY) ? 0.f : exp2f(x[nt][e] - m_run[half]);
        ps[nt][e] = p;
        rs[half] += p;
      }
#pragma unroll
    for (int half = 0; half < 2; ++half) l_run[half] = l_run[half] * alpha[half] + rs[half];
#pragma unroll
    for (int d = 0; d < kDTiles; ++d) {
      oc[d][0] *= alpha[0];
      oc[d][1] *= alpha[0];
      oc[d][2] *= alpha[1];
      oc[d][3] *= alpha[1];
    }
    uint32_t pa[4];
    pa[0] = pack2<T>(ps[0][0], ps[0][1]);
    pa[1] = pack2<T>(ps[0][2], ps[0][3]);
    pa[2] = pack2<T>(ps[1][0], ps[1][1]);
    pa[3] = pack2<T>(ps[1][2], ps[1][3]);

    // O += P V over the tile (V^T fragments via ldmatrix.trans).
#pragma unroll
    for (int d = 0; d < kDTiles; d += 2) {
      const int mtx = lane / 8, rr = lane % 8;
      const int key = ((mtx & 1) << 3) + rr;
      const int chunk = d + (mtx >> 1);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(vs + (uint32_t)(key * kChunks + (chunk ^ (key & 7))) * 16, b0, b1, b2, b3);
      mma16816<T>(oc[d], pa, b0, b1);
      mma16816<T>(oc[d + 1], pa, b2, b3);
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncthreads();  // ring is reused below

  // Merge the warps' states: row sums over the quad first.
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    l_run[half] += __shfl_xor_sync(0xffffffffu, l_run[half], 1);
    l_run[half] += __shfl_xor_sync(0xffffffffu, l_run[half], 2);
  }
  float* so = reinterpret_cast<float*>(smem);        // [kWarps][kRows][D]
  float* sml = so + kWarps * kRows * D;               // [kWarps][kRows][2]
#pragma unroll
  for (int d = 0; d < kDTiles; ++d)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = grp + 8 * (e >> 1);
      const int col = d * 8 + 2 * t4 + (e & 1);
      so[(warp * kRows + r) * D + col] = oc[d][e];
    }
  if (t4 == 0) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int r = grp + 8 * half;
      sml[(warp * kRows + r) * 2 + 0] = m_run[half];
      sml[(warp * kRows + r) * 2 + 1] = l_run[half];
    }
  }
  __syncthreads();
  const long long pbase = (((long long)b * P.Hkv + kvh) * part.max_splits + s) * kRows;
  for (int x = threadIdx.x; x < R * D; x += blockDim.x) {
    const int r = x / D, col = x % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sml[(w * kRows + r) * 2]);
    float o = 0.f, L = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float mw = sml[(w * kRows + r) * 2];
        const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        o += f * so[(w * kRows + r) * D + col];
        L += f * sml[(w * kRows + r) * 2 + 1];
      }
    }
    part.o[(pbase + r) * D + col] = o;
    if (col == 0) {
      part.ml[(pbase + r) * 2 + 0] = M;
      part.ml[(pbase + r) * 2 + 1] = L;
    }
  }
}

// One warp per output row (b, t, h): merge the row's splits and normalise. Lane j holds the
// (m, l) of splits j, j + 32, ... so the maximum and the weights come from shuffles, and the
// partial O rows are then read with no dependence on a branch.
template <typename T, int D>
__global__ void decode_combine_kernel(Problem P, Partials part, T* __restrict__ out) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + warp;  // (b, t, h)
  const long long rows = (long long)P.B * P.Lq * P.H;
  if (row >= rows) return;
  const int h = (int)(row % P.H);
  const int t = (int)((row / P.H) % P.Lq);
  const int b = (int)(row / ((long long)P.H * P.Lq));
  const int idx = P.cache_index[b];
  T* orow = out + row * D;
  if (idx < 0 || idx > P.Lk - P.Lq) {
    // the sequence was skipped (reported by the cache update): NaN rows make that visible
#pragma unroll
    for (int u = 0; u < D / 32; ++u) orow[lane + 32 * u] = from_f32<T>(__int_as_float(0x7fc00000));
    return;
  }
  const int kvlen = idx + P.Lq;
  int n_splits = (kvlen + part.split - 1) / part.split;
  const int kvh = h / P.group, r = t * P.group + (h % P.group);
  // range-checked build: every split read lies inside the partials, every row inside a tile
  if (!SDPA_CHECKED(P.status, n_splits <= part.max_splits && r < kRows)) n_splits = 0;
  const long long pbase = ((long long)b * P.Hkv + kvh) * part.max_splits;
  float M = -INFINITY;
  for (int s = lane; s < n_splits; s += 32) M = fmaxf(M, part.ml[((pbase + s) * kRows + r) * 2]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  constexpr int kPer = D / 32;
  float o[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) o[u] = 0.f;
  float L = 0.f;
  if (M != -INFINITY) {
    for (int s0 = 0; s0 < n_splits; s0 += 32) {
      // weight of split s0 + lane
      float f = 0.f, lw = 0.f;
      if (s0 + lane < n_splits) {
        const long long pr = (pbase + s0 + lane) * kRows + r;
        const float ms = part.ml[pr * 2];
        f = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
        lw = f * part.ml[pr * 2 + 1];
      }
      L += lw;
      const int n = min(32, n_splits - s0);
#pragma unroll 4
      for (int j = 0; j < n; ++j) {
        const float fj = __shfl_sync(0xffffffffu, f, j);
        const float* po = part.o + ((pbase + s0 + j) * kRows + r) * D + lane;
#pragma unroll
        for (int u = 0; u < kPer; ++u) o[u] += fj * po[32 * u];
      }
    }
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) L += __shfl_xor_sync(0xffffffffu, L, x);
  }
  const float inv = (L > 0.f) ? 1.f / L : __int_as_float(0x7fc00000);  // no key: NaN
#pragma unroll
  for (int u = 0; u < kPer; ++u) orow[lane + 32 * u] = from_f32<T>(L > 0.f ? o[u] * inv : inv);
}

int sm_count() {
  static int n = [] {
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v > 0 ? v : 148;
  }();
  return n;
}

// Keys per split: long splits stream longer and leave fewer partials to combine, but the grid
// must still fill the GPU. The largest of 1024 / 512 / 256 keys that gives at least eight
// CTAs per SM over the cache capacity (the lengths themselves are on the device).
int pick_split(const Problem& P) {
  const long long pairs = (long long)P.B * P.Hkv;
  for (int split : {1024, 512}) {
    if (pairs * ((P.Lk + split - 1) / split) >= 8LL * sm_count()) return split;
  }
  return 256;
}

}  // namespace

bool decode_supported(const Problem& P) {
  if (P.dtype != SDPA_BF16 && P.dtype != SDPA_F16) return false;
  if (P.D != P.Dv || (P.D != 64 && P.D != 128)) return false;
  if (P.Lq * P.group > kRows) return false;
  if (P.bias || P.mask || P.bcls) return false;
  return true;
}

size_t decode_workspace_bytes(const Problem& P) {
  const int split = pick_split(P);
  const long long max_splits = (P.Lk + split - 1) / split;
  const long long n = (long long)P.B * P.Hkv * max_splits * kRows;
  return (size_t)(n * P.Dv * 4 + n * 2 * 4 + 256);
}

cudaError_t launch_decode(const Problem& P, const void* q, const void* k_cache, const void* v_cache,
                          void* out, void* ws_partials, cudaStream_t stream) {
  Partials part;
  part.split = pick_split(P);
  part.max_splits = (P.Lk + part.split - 1) / part.split;
  const long long n = (long long)P.B * P.Hkv * part.max_splits * kRows;
  part.o = static_cast<float*>(ws_partials);
  part.ml = part.o + n * P.Dv;
  if (P.B == 0 || P.Lq == 0) return cudaSuccess;
  const dim3 grid(part.max_splits, P.Hkv, P.B);
  const long long rows = (long long)P.B * P.Lq * P.H;
  const dim3 cgrid((unsigned)((rows + 3) / 4));
  cudaError_t err;
#define SDPA_DECODE_CASE(TT, DD)                                                               \
  {                                                                                            \
    const size_t ring = (size_t)kWarps * kStages * 2 * kTileKeys * DD * 2;                     \
    const size_t merge = (size_t)kWarps * kRows * (DD + 2) * 4;                                \
    const size_t smem = ring > merge ? ring : merge;                                           \
    err = cudaFuncSetAttribute(decode_split_kernel<TT, DD>,                                    \
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);        \
    if (err != cudaSuccess) return err;                                                        \
    decode_split_kernel<TT, DD><<<grid, kWarps * 32, smem, stream>>>(                          \
        P, (const TT*)q, (const TT*)k_cache, (const TT*)v_cache, part);                        \
    err = cudaGetLastError();                                                                  \
    if (err != cudaSuccess) return err;                                                        \
    decode_combine_kernel<TT, DD><<<cgrid, 128, 0, stream>>>(P, part, (TT*)out);               \
    return cudaGetLastError();                                                                 \
  }
  if (P.dtype == SDPA_BF16) {
    if (P.D == 128) SDPA_DECODE_CASE(__nv_bfloat16, 128)
    SDPA_DECODE_CASE(__nv_bfloat16, 64)
  } else {
    if (P.D == 128) SDPA_DECODE_CASE(__half, 128)
    SDPA_DECODE_CASE(__half, 64)
  }
#undef SDPA_DECODE_CASE
}

}  // namespace sdpa
