// Internal declarations shared by the host resolver (sdpa_api.cu) and the kernels.
// Nothing here is part of the public ABI in include/sdpa.h.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/sdpa.h"

namespace sdpa {

// Status word values written by kernels (first error wins, via atomicCAS from SDPA_OK).
constexpr int kStatusOk = SDPA_OK;

// A call with every host-side argument resolved and validated. Per-batch values that live on
// the device (lengths, offsets, cache indices) stay there and are resolved by the kernels.
struct Problem {
  int dtype;                 // sdpa_dtype of q/k/v/out
  int B, Lq, Lk, H, Hkv, D, Dv, group;
  float scale;               // resolved (1/sqrt(D) when NaN was given)
  float scale_log2;          // scale * log2(e)
  int causal;                // sdpa_causal
  int q_offset_scalar;
  const int32_t* q_offset;   // device [B] or null
  const int32_t* q_lengths;  // device [B] or null
  const int32_t* kv_lengths; // device [B] or null
  const int32_t* cache_index;  // decode: kv_len[b] = cache_index[b] + Lq; else null
  const void* bias;
  int bias_dtype;
  long long bs[4];           // bias strides (j, i, h, b) in elements
  const uint8_t* mask;
  long long ms[4];           // mask strides (j, i, h, b)
  // block info (null bcls when absent)
  const uint8_t* bcls;
  const int32_t* brow_count;
  const uint32_t* brow_list;
  const uint32_t* bbits;
  int bi_nheads, bi_nqb, bi_nkb, bi_bq, bi_bk;
  // packed sequences (q_segments / kv_segments): B is the number of segments and Lq / Lk the
  // longest segment (maxlen); q_start / kv_start hold the first row of each segment in the
  // packed arrays, B + 1 entries, the last one the total row count. Null for a padded batch.
  const int32_t* q_start;
  const int32_t* kv_start;
  int Lq_total, Lk_total;    // rows of the packed arrays
  // scaled_dot_product_attention_with_weights on the tcgen05 kernel: the forward pass writes
  // each row's log-sum-exp (log2 units, +inf for a row with no key or past q_lengths) to lse;
  // the weights pass reads it, writes the weights [B][H][Lq][Lk] and applies the dropout
  // (keep when the row's 16-bit draw >= drop_thr, then scale by inv_keep)
  float* lse;
  float lse_out_mul;  // the forward stores lse (log2 units) times this (ln 2: natural log); 1 by default
  float lse_in_mul;   // the gradient reads lse times this as log2 units (log2 e for a natural log)
  void* weights;
  unsigned long long drop_seed;
  unsigned drop_thr;
  float inv_keep;
  // the statistics pass also writes the zero weights of the key tiles past each query tile's
  // causal bound (set only when no row can lack a key, so that none of them is NaN)
  int stats_fill;
  // rotary embedding of the Q tiles in shared memory (sdpa_forward_rope): (cos, sin) of each
  // query row's angles as fp16 pairs, [B * Lq][D / 2] 32-bit words; null when not rotated
  const uint32_t* q_rope;
  int* status;               // device status word (never null when a kernel runs)
  unsigned long long wait_timeout_ns;  // bound on every mbarrier wait of the tcgen05 kernel
  int selftest_stall;                  // SDPA_FLAG_SELFTEST_STALL
};

// Per-batch values every kernel resolves the same way.
struct BatchInfo {
  int q_len;   // valid queries
  int kv_len;  // valid keys
  int offset;  // causal offset (query i attends keys j <= offset + i)
  bool skip;   // decode: the cache index is out of range, leave this sequence alone
  int q_rows;  // rows of this sequence in the query / output arrays (rows past it are not written)
  long long q0, k0;  // first row of this sequence in the (rows, heads, dim) view of q / out, k / v
};

// Records the message sdpa_last_error() returns on this host thread.
void set_last_error(const char* msg);

// sdpa_backward (lse null: the forward runs again for the row log-sum-exp) and
// sdpa_backward_lse (lse: the caller's, natural log, from sdpa_forward_lse).
sdpa_status backward(const sdpa_params* p, const void* q, const void* k, const void* v, const void* out,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv, float* dscale, void* ws,
                     size_t ws_bytes, cudaStream_t stream);

// sdpa_decode_with_cache. Every argument is checked before anything is queued; with
// clear_status the status word at the start of `ws` is then zeroed on `stream` before the
// kernels run (the allocation-free entry point, whose scratch keeps the previous call's bytes).
sdpa_status decode_with_cache(const sdpa_params* p, const void* q, const void* k_new, const void* v_new,
                              void* k_cache, void* v_cache, const int32_t* cache_index, void* out, void* ws,
                              size_t ws_bytes, cudaStream_t stream, bool clear_status);

// Launchers (each returns a cudaError_t from the launch).
cudaError_t launch_generic(const Problem& P, const void* q, const void* k, const void* v,
                           void* out, cudaStream_t stream);
cudaError_t launch_cache_update(void* k_cache, void* v_cache, const void* k_new,
                                const void* v_new, int esize, int d, int Hkv, int n_new,
                                int capacity, int B, const int32_t* index, int* status,
                                cudaStream_t stream);
size_t decode_workspace_bytes(const Problem& P);
bool decode_supported(const Problem& P);
cudaError_t launch_decode(const Problem& P, const void* q, const void* k_cache,
                          const void* v_cache, void* out, void* ws_partials,
                          cudaStream_t stream);
cudaError_t launch_block_classify(const uint8_t* mask, const long long ms[3], int H, int Lq,
                                  int Lk, int bq, int bk, uint8_t* cls, int32_t* count,
                                  uint32_t* list, uint32_t* bits, int* status,
                                  cudaStream_t stream);
// Packed sequences: writes the first row of each query and key/value segment (exclusive prefix
// sums of the lengths, clamped to the array rows; n + 1 entries each). A negative length, one
// above maxlen, or lengths that do not add up to the array rows set SDPA_ERR_DEVICE_CHECK.
cudaError_t launch_segment_starts(const int32_t* q_segments, const int32_t* kv_segments, int n,
                                  int maxlen, int q_total, int kv_total, int32_t* q_start,
                                  int32_t* kv_start, int* status, cudaStream_t stream);
// The fused gradient (dq, dk, dv, dscale): three SIMT kernels. `ws` holds the per-row
// log-sum-exp and delta = dout . out (backward_workspace_bytes).
size_t backward_workspace_bytes(const Problem& P);
cudaError_t launch_backward(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                            const void* dout, void* dq, void* dk, void* dv, float* dscale, void* ws,
                            cudaStream_t stream);
// The same on mma.sync tiles (bf16 / fp16, head_dim = v_head_dim = 64 or 128); same workspace.
bool backward_mma_supported(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                            const void* dout);
cudaError_t launch_backward_mma(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                                const void* dout, void* dq, void* dk, void* dv, float* dscale, void* ws,
                                cudaStream_t stream);
// The same on the tcgen05 tensor cores (bf16 / fp16, head_dim = v_head_dim = 128, no bias, mask,
// block info or packed sequences): delta, dK / dV per key tile, dQ / dscale per query tile.
// lse and delta are [B][H][Lq] floats; lse (log2 units) must already hold the forward's row
// log-sum-exp.
bool backward_sm100_supported(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                              const void* dout, const void* dq, const void* dk, const void* dv);
cudaError_t launch_backward_sm100(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                                  const void* dout, void* dq, void* dk, void* dv, float* dscale, float* lse,
                                  float* delta, cudaStream_t stream);
// scaled_dot_product_attention_with_weights with dropout: mma.sync tiles (bf16 / fp16,
// head_dim = v_head_dim = 64 or 128) or SIMT. Needs no workspace.
bool weights_mma_supported(const Problem& P, const void* q, const void* k, const void* v, const void* out);
cudaError_t launch_weights(const Problem& P, bool tiles, const void* q, const void* k, const void* v, void* out,
                           void* weights, double drop_p, unsigned long long seed, cudaStream_t stream);
// Rotary position embedding of [rows][nheads][d] rows (out may alias x).
cudaError_t launch_rope(int dtype, const void* x, void* out, long long rows, int nheads, int d,
                        const int32_t* positions, double base, cudaStream_t stream);
// (cos, sin) of the rotary angles of `rows` positions as fp16 pairs: table[rows][d / 2].
cudaError_t launch_rope_table(long long rows, int d, const int32_t* positions, double base, void* table,
                              cudaStream_t stream);
bool prefill_supported(const Problem& P, const void* q, const void* k, const void* v,
                       const void* out);
// scaled_dot_product_attention_with_weights on the tcgen05 kernel (bf16 / fp16, head_dim =
// v_head_dim = 64 or 128, no bias, mask or block info, kv_len a multiple of 8): the forward
// with the row log-sum-exp into P.lse, the zero / NaN weights of the key tiles no query tile
// visits, then the weights pass. P.lse, P.weights and the dropout fields must be set.
bool prefill_weights_supported(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                               const void* weights);
cudaError_t launch_prefill_weights(const Problem& P, const void* q, const void* k, const void* v, void* out,
                                   cudaStream_t stream, const char** error_message);
size_t prefill_workspace_bytes(const Problem& P);
cudaError_t launch_prefill(const Problem& P, const void* q, const void* k, const void* v,
                           void* out, void* ws_sched, cudaStream_t stream,
                           const char** error_message);

}  // namespace sdpa
