// Host side of the tcgen05 prefill kernel (prefill_sm100.cuh): which calls it takes, the TMA
// tensor maps of Q, K and V, and the launch of the bias / mask variant the call needs.
#include <algorithm>

#include "prefill_sm100.cuh"
#include "tma_map.h"

namespace sdpa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up at run time (the library does not link libcuda).
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// A (batch, seq, heads, dim) array as a 4-d tensor map; box = 64 dims x 128 rows, 128B swizzle
// (the K-major / MN-major operand layout the MMA descriptors assume). Rows past `seq` read 0.
bool make_map(CUtensorMap* m, const void* base, int dtype, int D, int heads, int seq, int batch) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)seq, (cuuint64_t)batch};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2, (cuuint64_t)seq * heads * D * 2};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = dtype == SDPA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return fn(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// The 16-bit bias as a 4-d tensor map (keys, queries, heads, batch) for the shared-memory bias
// tiles: box = 64 keys x 128 queries, 128B swizzle. A broadcast head / batch dimension
// (stride 0) becomes an extent-1 dimension read at coordinate 0. Needs the keys contiguous and
// queries not broadcast; returns false otherwise (the kernel then reads the bias directly).
bool make_bias_map(CUtensorMap* m, const Problem& P) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !P.bias || P.bias_dtype == SDPA_F32 || P.bs[0] != 1 || P.bs[1] <= 0) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)P.Lk, (cuuint64_t)P.Lq, (cuuint64_t)(P.bs[2] != 0 ? P.H : 1),
                              (cuuint64_t)(P.bs[3] != 0 ? P.B : 1)};
  // an extent-1 (broadcast) dimension gets the packed stride after the previous dimension
  const long long row = P.bs[1] * 2;
  const long long sh = P.bs[2] != 0 ? P.bs[2] * 2 : row * P.Lq;
  const long long sb = P.bs[3] != 0 ? P.bs[3] * 2 : sh * (long long)dims[2];
  if (row % 16 || sh % 16 || sb % 16 || row <= 0 || sh <= 0 || sb <= 0) return false;
  const cuuint64_t strides[3] = {(cuuint64_t)row, (cuuint64_t)sh, (cuuint64_t)sb};
  const cuuint32_t box[4] = {64, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = P.dtype == SDPA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return fn(m, dt, 4, const_cast<void*>(P.bias), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

bool prefill_supported(const Problem& P, const void* q, const void* k, const void* v, const void* out) {
  if (P.dtype != SDPA_BF16 && P.dtype != SDPA_F16) return false;
  if (P.D != P.Dv || (P.D != 64 && P.D != 128)) return false;
  if (P.Lq <= 0 || P.Lk <= 0 || P.B <= 0) return false;
  if (!(P.scale > 0.f)) return false;  // the row max is taken on scaled logits
  if (P.bcls && (P.bi_bq != prefill::kBlockM || P.bi_bk != prefill::kBlockN)) return false;
  if ((long long)P.B * P.H * ((P.Lq + 127) / 128) >= (1LL << 30)) return false;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return false;
  if (P.bias) {
    // contiguous along keys, 16-byte aligned rows; the bias type is the input type or fp32
    const int es = P.bias_dtype == SDPA_F32 ? 4 : 2;
    if (P.bias_dtype != SDPA_F32 && P.bias_dtype != P.dtype) return false;
    if (P.bs[0] != 1 || !aligned(P.bias, 16)) return false;
    for (int d = 1; d < 4; ++d)
      if ((P.bs[d] * es) % 16 != 0) return false;
  }
  if (P.mask && !P.bcls) {
    if (P.ms[0] != 1 || !aligned(P.mask, 16)) return false;
    for (int d = 1; d < 4; ++d)
      if (P.ms[d] % 16 != 0) return false;
  }
  return encode_fn() != nullptr;
}

size_t prefill_workspace_bytes(const Problem&) { return 0; }

bool prefill_weights_supported(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                               const void* weights) {
  return !P.bias && !P.mask && !P.bcls && !P.q_start && P.Lk % 8 == 0 && aligned(weights, 16) &&
         prefill_supported(P, q, k, v, out);
}

// The weights as a 4-d tensor map (keys, queries, heads, batch), box 64 keys x `rows` queries in
// the 128-byte swizzle: 128 rows for the statistics pass's zero tile, 32 for the weights pass's
// stores (one warp's rows).
bool make_weights_map(CUtensorMap* m, const Problem& P, unsigned rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)P.Lk, (cuuint64_t)P.Lq, (cuuint64_t)P.H, (cuuint64_t)P.B};
  const cuuint64_t strides[3] = {(cuuint64_t)P.Lk * 2, (cuuint64_t)P.Lq * P.Lk * 2, (cuuint64_t)P.H * P.Lq * P.Lk * 2};
  const cuuint32_t box[4] = {64, rows, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = P.dtype == SDPA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return fn(m, dt, 4, P.weights, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_prefill_weights(const Problem& P0, const void* q, const void* k, const void* v, void* out,
                                   cudaStream_t stream, const char** msg) {
  // Every row has a key (so no weight is NaN) when no kv_lengths cut the keys and the causal
  // bound lets row 0 see key 0: then the statistics pass also writes the zero weights of the
  // key tiles past each query tile's bound, and the fill kernel is not needed.
  Problem P = P0;
  const bool rows_have_keys =
      P.kv_lengths == nullptr && P.Lk > 0 &&
      (P.causal == SDPA_CAUSAL_NONE || (P.causal == SDPA_CAUSAL_TOP_LEFT && P.q_offset == nullptr && P.q_offset_scalar >= 0) ||
       (P.causal == SDPA_CAUSAL_BOTTOM_RIGHT && P.Lk >= P.Lq));
  // 1. each row's log-sum-exp into P.lse (statistics only: the weights pass writes out)
  prefill::TensorMaps maps{};
  if (!make_map(&maps.q, q, P.dtype, P.D, P.H, P.Lq, P.B) || !make_map(&maps.k, k, P.dtype, P.D, P.Hkv, P.Lk, P.B) ||
      !make_map(&maps.v, v, P.dtype, P.D, P.Hkv, P.Lk, P.B) || !make_weights_map(&maps.w, P, 128) ||
      !make_weights_map(&maps.w_warp, P, 32)) {
    if (msg) *msg = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  P.stats_fill = rows_have_keys ? 1 : 0;
  const long long n_units = (long long)prefill::units_per_level(P) * prefill::n_levels(P);
  const int grid = (int)std::min<long long>(n_units, sm_count());
  cudaError_t e;
  if (P.dtype == SDPA_BF16)
    e = P.D == 128 ? prefill::launch_stats<__nv_bfloat16, 128>(maps, P, out, grid, stream)
                   : prefill::launch_stats<__nv_bfloat16, 64>(maps, P, out, grid, stream);
  else
    e = P.D == 128 ? prefill::launch_stats<__half, 128>(maps, P, out, grid, stream)
                   : prefill::launch_stats<__half, 64>(maps, P, out, grid, stream);
  if (e != cudaSuccess) {
    if (msg) *msg = "statistics pass launch";
    return e;
  }
  // 2. the weights of the key tiles the weights pass does not visit (unless the statistics pass
  // wrote them)
  if (!P.stats_fill) {
    const dim3 fgrid((unsigned)((P.Lq + prefill::kBlockM - 1) / prefill::kBlockM), (unsigned)P.H, (unsigned)P.B);
    if (P.dtype == SDPA_BF16)
      prefill::weights_fill_kernel<__nv_bfloat16><<<fgrid, 256, 0, stream>>>(P);
    else
      prefill::weights_fill_kernel<__half><<<fgrid, 256, 0, stream>>>(P);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
      if (msg) *msg = "weights fill launch";
      return e;
    }
  }
  // 3. the weights pass
  if (P.dtype == SDPA_BF16)
    e = P.D == 128 ? prefill::launch_weights<__nv_bfloat16, 128>(maps, P, out, grid, stream)
                   : prefill::launch_weights<__nv_bfloat16, 64>(maps, P, out, grid, stream);
  else
    e = P.D == 128 ? prefill::launch_weights<__half, 128>(maps, P, out, grid, stream)
                   : prefill::launch_weights<__half, 64>(maps, P, out, grid, stream);
  if (e != cudaSuccess && msg) *msg = "weights pass launch";
  return e;
}

cudaError_t launch_prefill(const Problem& P, const void* q, const void* k, const void* v, void* out, void*,
                           cudaStream_t stream, const char** msg) {
  prefill::TensorMaps maps{};
  // packed sequences: one batch of all rows, each sequence read from its own first row
  const bool packed = P.q_start != nullptr;
  const int q_rows = packed ? P.Lq_total : P.Lq, kv_rows = packed ? P.Lk_total : P.Lk, nb = packed ? 1 : P.B;
  if (!make_map(&maps.q, q, P.dtype, P.D, P.H, q_rows, nb) || !make_map(&maps.k, k, P.dtype, P.D, P.Hkv, kv_rows, nb) ||
      !make_map(&maps.v, v, P.dtype, P.D, P.Hkv, kv_rows, nb) || !make_map(&maps.o, out, P.dtype, P.D, P.H, q_rows, nb)) {
    if (msg) *msg = "cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  const bool bias_tiles = P.D == 64 && make_bias_map(&maps.bias, P);
  const long long n_units = (long long)prefill::units_per_level(P) * prefill::n_levels(P);
  const int grid = (int)std::min<long long>(n_units, sm_count());
  cudaError_t e;
  if (P.lse || P.q_rope) {
    // the forward with its row log-sum-exp and / or rotated Q tiles (no bias or mask: checked by
    // the callers)
    if (P.dtype == SDPA_BF16)
      e = P.D == 128 ? prefill::launch_aux<__nv_bfloat16, 128>(maps, P, out, grid, stream)
                     : prefill::launch_aux<__nv_bfloat16, 64>(maps, P, out, grid, stream);
    else
      e = P.D == 128 ? prefill::launch_aux<__half, 128>(maps, P, out, grid, stream)
                     : prefill::launch_aux<__half, 64>(maps, P, out, grid, stream);
    if (e != cudaSuccess && msg) *msg = "prefill launch";
    return e;
  }
  if (P.dtype == SDPA_BF16)
    e = P.D == 128 ? prefill::launch<__nv_bfloat16, 128>(maps, P, out, grid, false, stream)
                   : prefill::launch<__nv_bfloat16, 64>(maps, P, out, grid, bias_tiles, stream);
  else
    e = P.D == 128 ? prefill::launch<__half, 128>(maps, P, out, grid, false, stream)
                   : prefill::launch<__half, 64>(maps, P, out, grid, bias_tiles, stream);
  if (e != cudaSuccess && msg) *msg = "prefill launch";
  return e;
}

}  // namespace sdpa
