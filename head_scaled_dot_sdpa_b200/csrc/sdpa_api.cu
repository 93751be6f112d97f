// C ABI of libsdpa.so (declared in include/sdpa.h): argument validation, resolution of the
// defaults the Flux.jl page "Neural Network primitives from NNlib.jl" gives for
// scaled_dot_product_attention (scale = 1/sqrt(qk_head_dim), :bottom_right offsets, full
// lengths), kernel choice and launch. Nothing here reads device memory or synchronises, except
// sdpa_read_device_status, which exists for tests.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "internal.h"

namespace {

thread_local std::string g_last_error;
thread_local const char* g_last_kernel = "none";

constexpr size_t kStatusBytes = 256;

sdpa_status fail(sdpa_status code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
sdpa_status fail(sdpa_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

sdpa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SDPA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool valid_dtype(int d) { return d == SDPA_F32 || d == SDPA_F16 || d == SDPA_BF16; }
int dtype_size(int d) { return d == SDPA_F32 ? 4 : 2; }

// Validates the shape and optional arguments of a call and fills the resolved problem.
sdpa_status resolve(const sdpa_params* p, sdpa::Problem* P) {
  if (!p) return fail(SDPA_ERR_INVALID_ARG, "params is NULL");
  if (!valid_dtype(p->dtype)) return fail(SDPA_ERR_INVALID_ARG, "dtype %d is not an sdpa_dtype", (int)p->dtype);
  if (p->batch < 0 || p->q_len < 0 || p->kv_len < 0)
    return fail(SDPA_ERR_INVALID_ARG, "negative batch/q_len/kv_len");
  if (p->nheads <= 0 || p->nkvheads <= 0 || p->dqk <= 0 || p->dv <= 0)
    return fail(SDPA_ERR_INVALID_ARG, "nheads, nkvheads, dqk and dv must be positive");
  if (p->nheads % p->nkvheads != 0)
    return fail(SDPA_ERR_INVALID_ARG,
                "nheads (%d) must be divisible by nkvheads (%d) for grouped-query attention",
                p->nheads, p->nkvheads);
  if (p->causal < SDPA_CAUSAL_NONE || p->causal > SDPA_CAUSAL_BOTTOM_RIGHT)
    return fail(SDPA_ERR_INVALID_ARG, "causal %d is not an sdpa_causal", (int)p->causal);
  if (p->bias) {
    if (!valid_dtype(p->bias_dtype)) return fail(SDPA_ERR_INVALID_ARG, "bias_dtype is not an sdpa_dtype");
    for (int d = 0; d < 4; ++d)
      if (p->bias_stride[d] < 0) return fail(SDPA_ERR_INVALID_ARG, "negative bias stride");
  }
  if (p->mask)
    for (int d = 0; d < 4; ++d)
      if (p->mask_stride[d] < 0) return fail(SDPA_ERR_INVALID_ARG, "negative mask stride");
  const sdpa_block_mask_info* bi = p->block_info;
  if (bi) {
    if (!bi->block_class || !bi->row_count || !bi->row_list || !bi->partial_bits)
      return fail(SDPA_ERR_INVALID_ARG, "block_info has NULL arrays");
    if (bi->q_len != p->q_len || bi->kv_len != p->kv_len)
      return fail(SDPA_ERR_INVALID_ARG, "block_info was built for %dx%d, the call is %dx%d",
                  bi->q_len, bi->kv_len, p->q_len, p->kv_len);
    if (bi->nheads != 1 && bi->nheads != p->nheads)
      return fail(SDPA_ERR_INVALID_ARG, "block_info has %d heads, the call %d", bi->nheads, p->nheads);
    if (bi->bq <= 0 || bi->bk <= 0 || bi->bk % 32 != 0 ||
        bi->nqb != (p->q_len + bi->bq - 1) / bi->bq || bi->nkb != (p->kv_len + bi->bk - 1) / bi->bk)
      return fail(SDPA_ERR_INVALID_ARG, "block_info block sizes are inconsistent");
  }
  std::memset(P, 0, sizeof(*P));
  P->dtype = p->dtype;
  P->B = p->batch;
  P->Lq = p->q_len;
  P->Lk = p->kv_len;
  P->H = p->nheads;
  P->Hkv = p->nkvheads;
  P->D = p->dqk;
  P->Dv = p->dv;
  P->group = p->nheads / p->nkvheads;
  P->scale = std::isnan(p->scale) ? (float)(1.0 / std::sqrt((double)p->dqk)) : p->scale;
  P->scale_log2 = (float)((double)P->scale * 1.4426950408889634);
  P->causal = p->causal;
  P->q_offset_scalar = p->q_offset_scalar;
  P->q_offset = p->q_offset;
  P->q_lengths = p->q_lengths;
  P->kv_lengths = p->kv_lengths;
  P->bias = p->bias;
  P->bias_dtype = p->bias_dtype;
  for (int d = 0; d < 4; ++d) {
    P->bs[d] = p->bias_stride[d];
    P->ms[d] = p->mask_stride[d];
  }
  P->mask = p->mask;
  P->lse_out_mul = 1.f;
  P->lse_in_mul = 1.f;
  P->wait_timeout_ns = 1000000000ull;  // 1 s: far beyond any legitimate wait
  if (p->flags & SDPA_FLAG_SELFTEST_STALL) {
    P->wait_timeout_ns = 1000000ull;  // 1 ms
    P->selftest_stall = 1;
  }
  if (bi) {
    P->bcls = bi->block_class;
    P->brow_count = bi->row_count;
    P->brow_list = bi->row_list;
    P->bbits = bi->partial_bits;
    P->bi_nheads = bi->nheads;
    P->bi_nqb = bi->nqb;
    P->bi_nkb = bi->nkb;
    P->bi_bq = bi->bq;
    P->bi_bk = bi->bk;
  }
  return SDPA_OK;
}

sdpa_status check_workspace(void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(SDPA_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0)
    return fail(SDPA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < need) return fail(SDPA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  return SDPA_OK;
}

bool generic_ok(const sdpa::Problem& P) { return P.D <= 1024 && P.Dv <= 256; }

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

namespace sdpa {
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace sdpa

extern "C" {

size_t sdpa_workspace_size(const sdpa_params* p) {
  sdpa::Problem P;
  if (resolve(p, &P) != SDPA_OK) return 0;
  size_t extra = sdpa::prefill_workspace_bytes(P);
  if (sdpa::decode_supported(P)) {
    const size_t d = sdpa::decode_workspace_bytes(P);
    if (d > extra) extra = d;
  }
  return kStatusBytes + round256(extra);
}

sdpa_status sdpa_workspace_init(void* ws, size_t ws_bytes, struct CUstream_st* stream) {
  sdpa_status st = check_workspace(ws, ws_bytes, kStatusBytes);
  if (st != SDPA_OK) return st;
  cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync of the status word");
  return SDPA_OK;
}

sdpa_status sdpa_forward(const sdpa_params* p, const void* q, const void* k, const void* v,
                         void* out, void* ws, size_t ws_bytes, struct CUstream_st* stream) {
  sdpa::Problem P;
  sdpa_status st = resolve(p, &P);
  if (st != SDPA_OK) return st;
  const size_t need = sdpa_workspace_size(p);
  st = check_workspace(ws, ws_bytes, need);
  if (st != SDPA_OK) return st;
  if ((long long)P.B * P.Lq * P.H == 0) return SDPA_OK;
  if (!q || !out || (P.Lk > 0 && (!k || !v)))
    return fail(SDPA_ERR_INVALID_ARG, "q, k, v and out must not be NULL");
  P.status = static_cast<int*>(ws);
  void* scratch = static_cast<char*>(ws) + kStatusBytes;
  cudaStream_t s = (cudaStream_t)stream;
  if (!(p->flags & SDPA_FLAG_GENERIC_KERNEL) && sdpa::prefill_supported(P, q, k, v, out)) {
    const char* msg = nullptr;
    cudaError_t e = sdpa::launch_prefill(P, q, k, v, out, scratch, s, &msg);
    if (e != cudaSuccess) return cuda_fail(e, msg ? msg : "prefill launch");
    g_last_kernel = "prefill_tcgen05";
    return SDPA_OK;
  }
  if (!generic_ok(P))
    return fail(SDPA_ERR_UNSUPPORTED, "head sizes dqk=%d dv=%d exceed the SIMT kernel's limits (1024, 256)",
                P.D, P.Dv);
  cudaError_t e = sdpa::launch_generic(P, q, k, v, out, s);
  if (e != cudaSuccess) return cuda_fail(e, "generic attention launch");
  g_last_kernel = "generic_simt";
  return SDPA_OK;
}

sdpa_status sdpa_forward_lse(const sdpa_params* p, const void* q, const void* k, const void* v, void* out,
                             float* lse, void* ws, size_t ws_bytes, struct CUstream_st* stream) {
  sdpa::Problem P;
  sdpa_status st = resolve(p, &P);
  if (st != SDPA_OK) return st;
  st = check_workspace(ws, ws_bytes, sdpa_workspace_size(p));
  if (st != SDPA_OK) return st;
  if ((long long)P.B * P.Lq * P.H == 0) return SDPA_OK;
  if (!q || !out || !lse || (P.Lk > 0 && (!k || !v)))
    return fail(SDPA_ERR_INVALID_ARG, "q, k, v, out and lse must not be NULL");
  if ((p->flags & SDPA_FLAG_GENERIC_KERNEL) || P.bias || P.mask || P.bcls || !sdpa::prefill_supported(P, q, k, v, out))
    return fail(SDPA_ERR_UNSUPPORTED,
                "the row log-sum-exp comes from the tcgen05 kernel: bf16/fp16, qk_head_dim = v_head_dim = 64 or 128, "
                "no bias, mask or block_info");
  P.status = static_cast<int*>(ws);
  P.lse = lse;
  P.lse_out_mul = 0.69314718055994531f;  // natural log
  const char* msg = nullptr;
  cudaError_t e = sdpa::launch_prefill(P, q, k, v, out, nullptr, (cudaStream_t)stream, &msg);
  if (e != cudaSuccess) return cuda_fail(e, msg ? msg : "prefill launch");
  g_last_kernel = "prefill_tcgen05";
  return SDPA_OK;
}

}  // extern "C"

namespace {

// The packed call as a problem over nseg sequences of at most maxlen rows; the segment starts
// go in the workspace after the status word.
sdpa_status resolve_packed(const sdpa_params* p, const sdpa_packed_segments* seg, sdpa::Problem* P,
                           size_t* need) {
  sdpa_status st = resolve(p, P);
  if (st != SDPA_OK) return st;
  if (!seg) return fail(SDPA_ERR_INVALID_ARG, "segments are NULL");
  if (p->batch != 1)
    return fail(SDPA_ERR_INVALID_ARG, "packed sequences have no batch axis: batch must be 1, got %d", p->batch);
  if (p->bias || p->mask || p->block_info)
    return fail(SDPA_ERR_INVALID_ARG, "a bias or a mask is not supported with packed sequences");
  if (seg->nseg < 0 || seg->maxlen < 0) return fail(SDPA_ERR_INVALID_ARG, "negative nseg or maxlen");
  if (seg->nseg > 0 && !seg->q_segments) return fail(SDPA_ERR_INVALID_ARG, "q_segments is NULL");
  if (seg->nseg == 0 && (p->q_len > 0 || p->kv_len > 0))
    return fail(SDPA_ERR_INVALID_ARG, "no segments for %d query and %d key rows", p->q_len, p->kv_len);
  P->Lq_total = p->q_len;
  P->Lk_total = p->kv_len;
  P->B = seg->nseg;
  P->Lq = seg->maxlen;
  P->Lk = seg->maxlen;
  *need = kStatusBytes + round256(sdpa::prefill_workspace_bytes(*P)) +
          round256(2 * sizeof(int32_t) * ((size_t)seg->nseg + 1));
  return SDPA_OK;
}

}  // namespace

extern "C" {

size_t sdpa_packed_workspace_size(const sdpa_params* p, const sdpa_packed_segments* seg) {
  sdpa::Problem P;
  size_t need = 0;
  if (resolve_packed(p, seg, &P, &need) != SDPA_OK) return 0;
  return need;
}

sdpa_status sdpa_forward_packed(const sdpa_params* p, const sdpa_packed_segments* seg,
                                const void* q, const void* k, const void* v, void* out,
                                void* ws, size_t ws_bytes, struct CUstream_st* stream) {
  sdpa::Problem P;
  size_t need = 0;
  sdpa_status st = resolve_packed(p, seg, &P, &need);
  if (st != SDPA_OK) return st;
  st = check_workspace(ws, ws_bytes, need);
  if (st != SDPA_OK) return st;
  if (P.Lq_total == 0) return SDPA_OK;
  if (!q || !out || (P.Lk_total > 0 && (!k || !v)))
    return fail(SDPA_ERR_INVALID_ARG, "q, k, v and out must not be NULL");
  P.status = static_cast<int*>(ws);
  void* scratch = static_cast<char*>(ws) + kStatusBytes;
  int32_t* starts = reinterpret_cast<int32_t*>(static_cast<char*>(scratch) +
                                               round256(sdpa::prefill_workspace_bytes(P)));
  P.q_start = starts;
  P.kv_start = starts + P.B + 1;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = sdpa::launch_segment_starts(seg->q_segments, seg->kv_segments ? seg->kv_segments : seg->q_segments,
                                              P.B, seg->maxlen, P.Lq_total, P.Lk_total, starts, starts + P.B + 1,
                                              P.status, s);
  if (e != cudaSuccess) return cuda_fail(e, "segment scan launch");
  if (P.Lq == 0) return SDPA_OK;  // maxlen 0: every segment is empty (or flagged by the scan)
  if (!(p->flags & SDPA_FLAG_GENERIC_KERNEL) && P.Lk_total > 0 && sdpa::prefill_supported(P, q, k, v, out)) {
    const char* msg = nullptr;
    e = sdpa::launch_prefill(P, q, k, v, out, scratch, s, &msg);
    if (e != cudaSuccess) return cuda_fail(e, msg ? msg : "prefill launch");
    g_last_kernel = "prefill_tcgen05";
    return SDPA_OK;
  }
  if (!generic_ok(P))
    return fail(SDPA_ERR_UNSUPPORTED, "head sizes dqk=%d dv=%d exceed the SIMT kernel's limits (1024, 256)",
                P.D, P.Dv);
  e = sdpa::launch_generic(P, q, k, v, out, s);
  if (e != cudaSuccess) return cuda_fail(e, "generic attention launch");
  g_last_kernel = "generic_simt";
  return SDPA_OK;
}

size_t sdpa_weights_workspace_size(const sdpa_params* p) {
  sdpa::Problem P;
  if (resolve(p, &P) != SDPA_OK) return 0;
  return kStatusBytes + round256((size_t)P.B * P.H * P.Lq * sizeof(float));
}

sdpa_status sdpa_forward_with_weights(const sdpa_params* p, double drop_p, uint64_t seed, const void* q,
                                      const void* k, const void* v, void* out, void* weights, void* ws,
                                      size_t ws_bytes, struct CUstream_st* stream) {
  sdpa::Problem P;
  sdpa_status st = resolve(p, &P);
  if (st != SDPA_OK) return st;
  if (!(drop_p >= 0.0 && drop_p < 1.0)) return fail(SDPA_ERR_INVALID_ARG, "drop probability %g is not in [0, 1)", drop_p);
  if (P.Dv > 256) return fail(SDPA_ERR_UNSUPPORTED, "v_head_dim %d exceeds the weights kernels' limit (256)", P.Dv);
  if (P.D > 1024) return fail(SDPA_ERR_UNSUPPORTED, "head_dim %d exceeds the weights kernels' limit (1024)", P.D);
  st = check_workspace(ws, ws_bytes, sdpa_weights_workspace_size(p));
  if (st != SDPA_OK) return st;
  if ((long long)P.B * P.Lq * P.H == 0) return SDPA_OK;
  if (!q || !out || !weights || (P.Lk > 0 && (!k || !v)))
    return fail(SDPA_ERR_INVALID_ARG, "q, k, v, out and weights must not be NULL");
  P.status = static_cast<int*>(ws);
  if (!(p->flags & SDPA_FLAG_GENERIC_KERNEL) && P.Lk > 0 &&
      sdpa::prefill_weights_supported(P, q, k, v, out, weights)) {
    // tcgen05: the forward (with the row log-sum-exp in the workspace), the weights of the
    // unvisited key tiles, then the weights pass
    P.lse = reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes);
    P.weights = weights;
    P.drop_seed = (unsigned long long)seed;
    P.drop_thr = drop_p > 0.0 ? (unsigned)std::ceil(drop_p * 65536.0) : 0u;
    P.inv_keep = (float)(1.0 / (1.0 - drop_p));
    const char* msg = nullptr;
    cudaError_t e = sdpa::launch_prefill_weights(P, q, k, v, out, (cudaStream_t)stream, &msg);
    if (e != cudaSuccess) return cuda_fail(e, msg ? msg : "weights launch");
    g_last_kernel = "weights_tcgen05";
    return SDPA_OK;
  }
  const bool tiles = !(p->flags & SDPA_FLAG_GENERIC_KERNEL) && P.Lk > 0 && sdpa::weights_mma_supported(P, q, k, v, out);
  cudaError_t e = sdpa::launch_weights(P, tiles, q, k, v, out, weights, drop_p, (unsigned long long)seed,
                                       (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "weights launch");
  g_last_kernel = tiles ? "weights_mma" : "weights_simt";
  return SDPA_OK;
}

sdpa_status sdpa_rope(const void* x, void* out, sdpa_dtype dtype, int64_t rows, int32_t nheads, int32_t d,
                      const int32_t* positions, double base, struct CUstream_st* stream) {
  if (!valid_dtype(dtype)) return fail(SDPA_ERR_INVALID_ARG, "dtype is not an sdpa_dtype");
  if (rows < 0 || nheads <= 0 || d <= 0 || d % 2 != 0)
    return fail(SDPA_ERR_INVALID_ARG, "rotary embedding needs rows >= 0, nheads > 0 and an even head size (got %d)", d);
  if (!(base > 0.0)) return fail(SDPA_ERR_INVALID_ARG, "rotary base must be positive");
  if (d > 8192) return fail(SDPA_ERR_UNSUPPORTED, "rotary embedding supports head sizes up to 8192 (got %d)", d);
  if (rows == 0) return SDPA_OK;
  if (!x || !out || !positions) return fail(SDPA_ERR_INVALID_ARG, "x, out and positions must not be NULL");
  cudaError_t e = sdpa::launch_rope(dtype, x, out, rows, nheads, d, positions, base, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "rotary embedding launch");
  return SDPA_OK;
}

// Workspace of sdpa_forward_rope: the status word, then the rotated keys, the cos / sin table
// of the query rows (the tcgen05 kernel rotates its Q tiles with it) and room for rotated
// queries (the other kernels take them from memory).
namespace {
struct RopeLayout {
  size_t k_off, table_off, q_off, total;
};
RopeLayout rope_layout(const sdpa::Problem& P) {
  RopeLayout L;
  const size_t es = P.dtype == SDPA_F32 ? 4 : 2;
  L.k_off = kStatusBytes;
  L.table_off = L.k_off + round256((size_t)P.B * P.Lk * P.Hkv * P.D * es);
  L.q_off = L.table_off + round256((size_t)P.B * P.Lq * (P.D / 2) * sizeof(uint32_t));
  L.total = L.q_off + round256((size_t)P.B * P.Lq * P.H * P.D * es) +
            round256(sdpa::prefill_workspace_bytes(P));
  return L;
}
}  // namespace

size_t sdpa_rope_workspace_size(const sdpa_params* p) {
  sdpa::Problem P;
  if (resolve(p, &P) != SDPA_OK || P.D % 2 != 0) return 0;
  return rope_layout(P).total;
}

sdpa_status sdpa_forward_rope(const sdpa_params* p, const int32_t* q_positions, const int32_t* k_positions,
                              double base, const void* q, const void* k, const void* v, void* out, void* ws,
                              size_t ws_bytes, struct CUstream_st* stream) {
  sdpa::Problem P;
  sdpa_status st = resolve(p, &P);
  if (st != SDPA_OK) return st;
  if (P.D % 2 != 0 || P.D > 8192)
    return fail(SDPA_ERR_INVALID_ARG, "the rotary embedding needs an even qk_head_dim of at most 8192 (got %d)", P.D);
  if (!(base > 0.0)) return fail(SDPA_ERR_INVALID_ARG, "rotary base must be positive");
  const RopeLayout L = rope_layout(P);
  st = check_workspace(ws, ws_bytes, L.total);
  if (st != SDPA_OK) return st;
  if ((long long)P.B * P.Lq * P.H == 0) return SDPA_OK;
  if (!q || !out || (P.Lk > 0 && (!k || !v || !k_positions)) || !q_positions)
    return fail(SDPA_ERR_INVALID_ARG, "q, k, v, out and the positions must not be NULL");
  P.status = static_cast<int*>(ws);
  char* base_ws = static_cast<char*>(ws);
  void* k_rot = base_ws + L.k_off;
  cudaStream_t s = (cudaStream_t)stream;
  // the keys, rotated once: every query tile of the key/value head reads them
  cudaError_t e = sdpa::launch_rope(P.dtype, k, k_rot, (long long)P.B * P.Lk, P.Hkv, P.D, k_positions, base, s);
  if (e != cudaSuccess) return cuda_fail(e, "rotary embedding of the keys");
  if (!(p->flags & SDPA_FLAG_GENERIC_KERNEL) && !P.bias && !P.mask && !P.bcls &&
      sdpa::prefill_supported(P, q, k_rot, v, out)) {
    // the queries are rotated tile by tile in shared memory, from a cos / sin table
    void* table = base_ws + L.table_off;
    e = sdpa::launch_rope_table((long long)P.B * P.Lq, P.D, q_positions, base, table, s);
    if (e != cudaSuccess) return cuda_fail(e, "rotary table");
    P.q_rope = static_cast<const uint32_t*>(table);
    const char* msg = nullptr;
    e = sdpa::launch_prefill(P, q, k_rot, v, out, base_ws + L.q_off, s, &msg);
    if (e != cudaSuccess) return cuda_fail(e, msg ? msg : "prefill launch");
    g_last_kernel = "prefill_tcgen05_rope";
    return SDPA_OK;
  }
  void* q_rot = base_ws + L.q_off;
  e = sdpa::launch_rope(P.dtype, q, q_rot, (long long)P.B * P.Lq, P.H, P.D, q_positions, base, s);
  if (e != cudaSuccess) return cuda_fail(e, "rotary embedding of the queries");
  if (!(p->flags & SDPA_FLAG_GENERIC_KERNEL) && sdpa::prefill_supported(P, q_rot, k_rot, v, out)) {
    // a bias or a mask: the queries rotated into the workspace, then the tcgen05 forward
    const char* msg = nullptr;
    e = sdpa::launch_prefill(P, q_rot, k_rot, v, out, nullptr, s, &msg);
    if (e != cudaSuccess) return cuda_fail(e, msg ? msg : "prefill launch");
    g_last_kernel = "prefill_tcgen05";
    return SDPA_OK;
  }
  if (!generic_ok(P))
    return fail(SDPA_ERR_UNSUPPORTED, "head sizes dqk=%d dv=%d exceed the SIMT kernel's limits (1024, 256)",
                P.D, P.Dv);
  e = sdpa::launch_generic(P, q_rot, k_rot, v, out, s);
  if (e != cudaSuccess) return cuda_fail(e, "generic attention launch");
  g_last_kernel = "generic_simt";
  return SDPA_OK;
}

size_t sdpa_backward_workspace_size(const sdpa_params* p) {
  sdpa::Problem P;
  if (resolve(p, &P) != SDPA_OK) return 0;
  return kStatusBytes + round256(sdpa::backward_workspace_bytes(P));
}

sdpa_status sdpa_backward(const sdpa_params* p, const void* q, const void* k, const void* v,
                          const void* out, const void* dout, void* dq, void* dk, void* dv,
                          float* dscale, void* ws, size_t ws_bytes, struct CUstream_st* stream) {
  return sdpa::backward(p, q, k, v, out, dout, nullptr, dq, dk, dv, dscale, ws, ws_bytes, (cudaStream_t)stream);
}

sdpa_status sdpa_backward_lse(const sdpa_params* p, const void* q, const void* k, const void* v,
                              const void* out, const void* dout, const float* lse, void* dq, void* dk, void* dv,
                              float* dscale, void* ws, size_t ws_bytes, struct CUstream_st* stream) {
  if (!lse) return fail(SDPA_ERR_INVALID_ARG, "lse must not be NULL");
  return sdpa::backward(p, q, k, v, out, dout, lse, dq, dk, dv, dscale, ws, ws_bytes, (cudaStream_t)stream);
}

}  // extern "C"

namespace sdpa {

sdpa_status backward(const sdpa_params* p, const void* q, const void* k, const void* v, const void* out,
                     const void* dout, const float* lse_in, void* dq, void* dk, void* dv, float* dscale, void* ws,
                     size_t ws_bytes, cudaStream_t stream) {
  sdpa::Problem P;
  sdpa_status st = resolve(p, &P);
  if (st != SDPA_OK) return st;
  if (p->bias)
    return fail(SDPA_ERR_INVALID_ARG,
                "the fused gradient takes no bias (a call with a bias takes the materialized implementation)");
  if (P.D > 256 || P.Dv > 256)
    return fail(SDPA_ERR_UNSUPPORTED, "head sizes dqk=%d dv=%d exceed the gradient kernels' limit (256)", P.D, P.Dv);
  st = check_workspace(ws, ws_bytes, sdpa_backward_workspace_size(p));
  if (st != SDPA_OK) return st;
  if ((long long)P.B * P.Lq * P.H == 0 && (long long)P.B * P.Lk * P.Hkv == 0) return SDPA_OK;
  if (!q || !k || !v || !out || !dout || !dq || !dk || !dv)
    return fail(SDPA_ERR_INVALID_ARG, "q, k, v, out, dout, dq, dk and dv must not be NULL");
  P.status = static_cast<int*>(ws);
  void* scratch = static_cast<char*>(ws) + kStatusBytes;
  if (!(p->flags & SDPA_FLAG_GENERIC_KERNEL) && sdpa::backward_sm100_supported(P, q, k, v, out, dout, dq, dk, dv) &&
      sdpa::prefill_supported(P, q, k, v, dq)) {
    // tcgen05: the row log-sum-exp (the caller's, from sdpa_forward_lse, or the forward again,
    // whose output goes to dq, which the gradient overwrites), then delta, dK / dV and dQ / dscale
    float* lse = static_cast<float*>(scratch);
    float* delta = lse + (size_t)P.B * P.H * P.Lq;
    cudaError_t e = cudaSuccess;
    if (lse_in) {
      lse = const_cast<float*>(lse_in);
      P.lse_in_mul = 1.4426950408889634f;  // natural log -> log2 units
    } else {
      sdpa::Problem F = P;
      F.lse = lse;
      const char* msg = nullptr;
      e = sdpa::launch_prefill(F, q, k, v, dq, nullptr, (cudaStream_t)stream, &msg);
      if (e != cudaSuccess) return cuda_fail(e, msg ? msg : "prefill launch");
    }
    e = sdpa::launch_backward_sm100(P, q, k, v, out, dout, dq, dk, dv, dscale, lse, delta, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "gradient launch");
    g_last_kernel = "backward_tcgen05";
    return SDPA_OK;
  }
  if (!(p->flags & SDPA_FLAG_GENERIC_KERNEL) && sdpa::backward_mma_supported(P, q, k, v, out, dout)) {
    cudaError_t e = sdpa::launch_backward_mma(P, q, k, v, out, dout, dq, dk, dv, dscale, scratch, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "gradient launch");
    g_last_kernel = "backward_mma";
    return SDPA_OK;
  }
  cudaError_t e = sdpa::launch_backward(P, q, k, v, out, dout, dq, dk, dv, dscale, scratch, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "gradient launch");
  g_last_kernel = "backward_simt";
  return SDPA_OK;
}

}  // namespace sdpa

extern "C" {

sdpa_status cache_update_at_index(void* k_cache, void* v_cache, const void* k_new,
                                  const void* v_new, sdpa_dtype dtype, int32_t d,
                                  int32_t nkvheads, int32_t n_new, int32_t capacity,
                                  int32_t batch, const int32_t* index, void* ws,
                                  struct CUstream_st* stream) {
  if (!valid_dtype(dtype)) return fail(SDPA_ERR_INVALID_ARG, "dtype is not an sdpa_dtype");
  if (d <= 0 || nkvheads <= 0 || n_new < 0 || capacity < 0 || batch < 0)
    return fail(SDPA_ERR_INVALID_ARG, "invalid cache sizes");
  if (n_new > capacity) return fail(SDPA_ERR_INVALID_ARG, "n_new (%d) exceeds capacity (%d)", n_new, capacity);
  if (batch == 0 || n_new == 0) return SDPA_OK;
  if (!index) return fail(SDPA_ERR_INVALID_ARG, "index is NULL");
  if ((k_cache == nullptr) != (k_new == nullptr) || (v_cache == nullptr) != (v_new == nullptr))
    return fail(SDPA_ERR_INVALID_ARG, "each cache needs its new rows (or both NULL)");
  if (ws && reinterpret_cast<uintptr_t>(ws) % 256 != 0)
    return fail(SDPA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  cudaError_t e = sdpa::launch_cache_update(k_cache, v_cache, k_new, v_new, dtype_size(dtype), d,
                                            nkvheads, n_new, capacity, batch, index,
                                            static_cast<int*>(ws), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cache update launch");
  return SDPA_OK;
}

sdpa_status sdpa_decode_with_cache(const sdpa_params* p, const void* q, const void* k_new,
                                   const void* v_new, void* k_cache, void* v_cache,
                                   const int32_t* cache_index, void* out, void* ws,
                                   size_t ws_bytes, struct CUstream_st* stream) {
  return sdpa::decode_with_cache(p, q, k_new, v_new, k_cache, v_cache, cache_index, out, ws, ws_bytes,
                                 (cudaStream_t)stream, false);
}

}  // extern "C"

namespace sdpa {

sdpa_status decode_with_cache(const sdpa_params* p, const void* q, const void* k_new, const void* v_new,
                              void* k_cache, void* v_cache, const int32_t* cache_index, void* out, void* ws,
                              size_t ws_bytes, cudaStream_t s, bool clear_status) {
  sdpa::Problem P;
  sdpa_status st = resolve(p, &P);
  if (st != SDPA_OK) return st;
  if (p->causal != SDPA_CAUSAL_BOTTOM_RIGHT)
    return fail(SDPA_ERR_INVALID_ARG, "decode attends with causal = SDPA_CAUSAL_BOTTOM_RIGHT");
  if (p->q_lengths || p->kv_lengths || p->bias || p->mask || p->block_info)
    return fail(SDPA_ERR_INVALID_ARG,
                "decode takes its lengths from cache_index; q_lengths, kv_lengths, bias, mask "
                "and block_info must be NULL");
  if (P.Lq > P.Lk) return fail(SDPA_ERR_INVALID_ARG, "n_new (%d) exceeds capacity (%d)", P.Lq, P.Lk);
  const size_t need = sdpa_workspace_size(p);
  st = check_workspace(ws, ws_bytes, need);
  if (st != SDPA_OK) return st;
  if (P.B == 0 || P.Lq == 0) return SDPA_OK;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !cache_index || !out)
    return fail(SDPA_ERR_INVALID_ARG, "decode pointers must not be NULL");
  // every argument is valid: only now may the status word be cleared (a caller-owned
  // workspace keeps the caller's word as it is)
  cudaError_t e = clear_status ? cudaMemsetAsync(ws, 0, kStatusBytes, s) : cudaSuccess;
  if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  e = sdpa::launch_cache_update(k_cache, nullptr, k_new, nullptr, dtype_size(P.dtype), P.D,
                                            P.Hkv, P.Lq, P.Lk, P.B, cache_index, static_cast<int*>(ws), s);
  if (e == cudaSuccess)
    e = sdpa::launch_cache_update(nullptr, v_cache, nullptr, v_new, dtype_size(P.dtype), P.Dv, P.Hkv,
                                  P.Lq, P.Lk, P.B, cache_index, static_cast<int*>(ws), s);
  if (e != cudaSuccess) return cuda_fail(e, "cache update launch");
  P.cache_index = cache_index;
  P.status = static_cast<int*>(ws);
  void* scratch = static_cast<char*>(ws) + kStatusBytes;
  if (!(p->flags & SDPA_FLAG_GENERIC_KERNEL) && sdpa::decode_supported(P)) {
    e = sdpa::launch_decode(P, q, k_cache, v_cache, out, scratch, s);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    g_last_kernel = "decode_splitkv";
    return SDPA_OK;
  }
  if (!generic_ok(P)) return fail(SDPA_ERR_UNSUPPORTED, "head sizes exceed the SIMT kernel's limits");
  e = sdpa::launch_generic(P, q, k_cache, v_cache, out, s);
  if (e != cudaSuccess) return cuda_fail(e, "generic attention launch");
  g_last_kernel = "generic_simt";
  return SDPA_OK;
}

}  // namespace sdpa

extern "C" {

size_t build_block_mask_info_size(int32_t nheads, int32_t q_len, int32_t kv_len, int32_t bq,
                                  int32_t bk) {
  if (nheads <= 0 || q_len <= 0 || kv_len <= 0 || bq <= 0 || bk <= 0 || bk % 32 != 0) return 0;
  if ((long long)bq * (bk / 32) > 2048) return 0;
  const size_t nqb = (size_t)(q_len + bq - 1) / bq, nkb = (size_t)(kv_len + bk - 1) / bk;
  const size_t blocks = (size_t)nheads * nqb * nkb;
  return round256(blocks) + round256((size_t)nheads * nqb * 4) + round256(blocks * 4) +
         round256(blocks * (size_t)bq * (bk / 32) * 4);
}

sdpa_status build_block_mask_info(const uint8_t* mask, const int64_t mask_stride[3],
                                  int32_t nheads, int32_t q_len, int32_t kv_len, int32_t bq,
                                  int32_t bk, void* info_buf, size_t info_bytes,
                                  sdpa_block_mask_info* out_info, struct CUstream_st* stream) {
  const size_t need = build_block_mask_info_size(nheads, q_len, kv_len, bq, bk);
  if (need == 0)
    return fail(SDPA_ERR_INVALID_ARG,
                "invalid block mask sizes (need positive sizes, bk %% 32 == 0, bq*bk <= 65536)");
  if (!mask || !mask_stride || !out_info) return fail(SDPA_ERR_INVALID_ARG, "NULL mask, strides or out_info");
  if (mask_stride[0] != 1) return fail(SDPA_ERR_INVALID_ARG, "mask_stride[0] (keys) must be 1");
  if (mask_stride[1] < 0 || mask_stride[2] < 0) return fail(SDPA_ERR_INVALID_ARG, "negative mask stride");
  if (!info_buf || reinterpret_cast<uintptr_t>(info_buf) % 256 != 0)
    return fail(SDPA_ERR_WORKSPACE, "info buffer must be non-NULL and 256-byte aligned");
  if (info_bytes < need) return fail(SDPA_ERR_WORKSPACE, "info buffer has %zu bytes, needs %zu", info_bytes, need);
  const int nqb = (q_len + bq - 1) / bq, nkb = (kv_len + bk - 1) / bk;
  if (nqb > 65535 || nheads > 65535)
    return fail(SDPA_ERR_INVALID_ARG, "at most 65535 query blocks and 65535 mask heads (got %d, %d)", nqb, nheads);
  const size_t blocks = (size_t)nheads * nqb * nkb;
  char* base = static_cast<char*>(info_buf);
  uint8_t* cls = reinterpret_cast<uint8_t*>(base);
  int32_t* count = reinterpret_cast<int32_t*>(base + round256(blocks));
  uint32_t* list = reinterpret_cast<uint32_t*>(base + round256(blocks) + round256((size_t)nheads * nqb * 4));
  uint32_t* bits = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(list) + round256(blocks * 4));
  out_info->nheads = nheads;
  out_info->q_len = q_len;
  out_info->kv_len = kv_len;
  out_info->bq = bq;
  out_info->bk = bk;
  out_info->nqb = nqb;
  out_info->nkb = nkb;
  out_info->block_class = cls;
  out_info->row_count = count;
  out_info->row_list = list;
  out_info->partial_bits = bits;
  const long long ms[3] = {mask_stride[0], mask_stride[1], mask_stride[2]};
  cudaError_t e = sdpa::launch_block_classify(mask, ms, nheads, q_len, kv_len, bq, bk, cls, count, list,
                                              bits, nullptr, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "block classification launch");
  return SDPA_OK;
}

sdpa_status sdpa_read_device_status(void* ws, struct CUstream_st* stream) {
  if (!ws) return fail(SDPA_ERR_WORKSPACE, "workspace is NULL");
  cudaStream_t s = (cudaStream_t)stream;
  int status = 0;
  cudaError_t e = cudaMemcpyAsync(&status, ws, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(int), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  if (status != SDPA_OK) {
    g_last_error = "device reported an error in the status word";
    return (sdpa_status)status;
  }
  return SDPA_OK;
}

const char* sdpa_last_error(void) { return g_last_error.c_str(); }

const char* sdpa_last_kernel(void) { return g_last_kernel; }

int sdpa_debug_checks(void) {
#ifdef SDPA_DEBUG_CHECKS
  return 1;
#else
  return 0;
#endif
}

}  // extern "C"
