/*
 * sdpa.h — C ABI of libsdpa.so: multi-head scaled-dot-product attention on NVIDIA B200
 * (sm_100a): the forward pass, KV-cache decode, the gradient, the with-weights variant with
 * dropout, and the rotary embedding of query / key rows.
 *
 * The operation is NNlib.scaled_dot_product_attention as the Flux.jl page "Neural Network
 * primitives from NNlib.jl" defines it (entry "scaled_dot_product_attention", section
 * "Arguments"):
 *
 *     out = softmax(scale * query' * key + bias, masked) * value
 *
 * with grouped-query sharing of key/value heads, is_causal (top-left with q_offset, or
 * :bottom_right), per-batch q_lengths / kv_lengths, a broadcast additive bias and a boolean
 * mask, computed tile by tile with an online softmax (section "Fused implementation").
 *
 * Conventions for every call:
 *  - Layout. q, k, v and out are dense arrays in the page's column-major
 *    (head_dim, nheads, seq_len, batch) order, which is row-major [batch][seq][head][dim]:
 *      q   [batch][q_len ][nheads  ][dqk]
 *      k   [batch][kv_len][nkvheads][dqk]
 *      v   [batch][kv_len][nkvheads][dv ]
 *      out [batch][q_len ][nheads  ][dv ]
 *    Several trailing batch dimensions of the page are flattened into one `batch`.
 *  - Ownership. Every data pointer is a DEVICE pointer owned by the caller; the library keeps
 *    no reference after the call returns and allocates no device memory. Scratch space is a
 *    caller-owned workspace sized by sdpa_workspace_size().
 *  - Asynchrony. Calls enqueue work on `stream` and return without synchronising. Lengths and
 *    offsets that live on the device are never read on the host.
 *  - Errors. Invalid arguments are reported before anything is launched, as a status code;
 *    sdpa_last_error() gives a message. Errors found on the device (an out-of-range cache
 *    index, a bounded wait that ran out) are recorded in the workspace's status word and read
 *    with sdpa_read_device_status(). No call aborts the process or traps the GPU.
 */
#ifndef SDPA_H_
#define SDPA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t */

#if defined(__GNUC__)
#define SDPA_API __attribute__((visibility("default")))
#else
#define SDPA_API
#endif

typedef enum {
  SDPA_OK = 0,
  SDPA_ERR_INVALID_ARG = 1, /* shape, stride, pointer or enum out of range */
  SDPA_ERR_UNSUPPORTED = 2, /* valid request that no kernel here implements */
  SDPA_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or too small */
  SDPA_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
  SDPA_ERR_TIMEOUT = 5,     /* device: a bounded wait ran out (read via the status word) */
  SDPA_ERR_DEVICE_CHECK = 6 /* device: an index check failed, the access was skipped */
} sdpa_status;

typedef enum { SDPA_F32 = 0, SDPA_F16 = 1, SDPA_BF16 = 2 } sdpa_dtype;

/* Argument is_causal: false, true (query i attends keys j <= q_offset + i), or :bottom_right
 * (q_offset = kv_lengths - q_lengths, the array sizes standing in for lengths not given). */
typedef enum {
  SDPA_CAUSAL_NONE = 0,
  SDPA_CAUSAL_TOP_LEFT = 1,
  SDPA_CAUSAL_BOTTOM_RIGHT = 2
} sdpa_causal;

/* Block classes of a boolean mask (splash-attention mask info of the JAX pull request
 * "Support dynamic masks in splash attention"; this encoding is this library's own). */
enum { SDPA_BLOCK_EMPTY = 0, SDPA_BLOCK_PARTIAL = 1, SDPA_BLOCK_FULL = 2 };

/* Result of build_block_mask_info(); every pointer is into the caller's info buffer.
 *  block_class [nheads][nqb][nkb]     SDPA_BLOCK_* of each bq x bk block
 *  row_count   [nheads][nqb]          number of non-empty blocks in block row qb
 *  row_list    [nheads][nqb][nkb]     the first row_count entries: kb | (class << 30), kb
 *                                     increasing
 *  partial_bits[nheads][nqb][nkb][bq][bk/32]  for PARTIAL blocks only: bit c of word w of
 *                                     row r is mask(head, qb*bq + r, kb*bk + 32*w + c);
 *                                     cells past q_len / kv_len are 0.
 * nheads is the mask's own head extent (1 when it is broadcast over heads). */
typedef struct sdpa_block_mask_info {
  int32_t nheads, q_len, kv_len, bq, bk, nqb, nkb;
  const uint8_t* block_class;
  const int32_t* row_count;
  const uint32_t* row_list;
  const uint32_t* partial_bits;
} sdpa_block_mask_info;

/* Flags (sdpa_params.flags). */
#define SDPA_FLAG_GENERIC_KERNEL 0x1u /* force the SIMT kernel (any dtype / head size) */
/* Self-test of the bounded waits (tests only): every mbarrier wait of the tcgen05 kernel is
 * limited to 1 ms and its TMA producer first waits on a barrier that nothing completes, so the
 * call ends early with SDPA_ERR_TIMEOUT in the status word and the context stays usable. */
#define SDPA_FLAG_SELFTEST_STALL 0x2u

/* One attention call. Arguments of the page's entry and where they sit here:
 *  dtype            element type of q, k, v and out (fp32 accumulation throughout; out is
 *                   rounded to nearest even).
 *  batch, q_len, kv_len, nheads, nkvheads, dqk, dv   the array sizes. nheads % nkvheads must
 *                   be 0 (GQA paragraph); query head h uses key/value head
 *                   h / (nheads / nkvheads).
 *  scale            multiplier of query'*key; NaN means 1/sqrt(dqk) (argument `scale`).
 *  causal, q_offset_scalar, q_offset   argument `is_causal` and `q_offset`: q_offset is a
 *                   device int32[batch] or NULL for q_offset_scalar; ignored unless
 *                   causal == SDPA_CAUSAL_TOP_LEFT.
 *  q_lengths, kv_lengths   device int32[batch] or NULL (full length). Keys j >= kv_lengths[b]
 *                   are not attended; output rows i >= q_lengths[b] are zero. Values must
 *                   lie in [0, q_len] / [0, kv_len]. The tcgen05 kernel reads whole tiles of
 *                   128 keys, so the rows of k and v past kv_lengths[b], up to the next
 *                   multiple of 128 (or the array end), must hold finite values: they get a
 *                   weight of exactly 0, and 0 times Inf or NaN is NaN.
 *  bias             NULL or a device array of bias_dtype, element (key j, query i, head h,
 *                   batch b) at bias[j*bias_stride[0] + i*bias_stride[1] + h*bias_stride[2]
 *                   + b*bias_stride[3]]; a stride of 0 broadcasts (argument `bias`: added to
 *                   the logits, not scaled).
 *  mask             NULL or a device uint8 array (0 = not attended), addressed like the bias
 *                   with mask_stride (argument `mask`). mask, is_causal and kv_lengths
 *                   combine by AND.
 *  block_info       NULL, or the classification of `mask` built by build_block_mask_info;
 *                   then empty blocks are skipped and only partial blocks' bits are read
 *                   (`mask` may then be NULL). The mask it describes must not vary with batch.
 *  flags            SDPA_FLAG_* bits. */
typedef struct sdpa_params {
  sdpa_dtype dtype;
  int32_t batch, q_len, kv_len, nheads, nkvheads, dqk, dv;
  float scale;
  sdpa_causal causal;
  int32_t q_offset_scalar;
  const int32_t* q_offset;
  const int32_t* q_lengths;
  const int32_t* kv_lengths;
  const void* bias;
  sdpa_dtype bias_dtype;
  int64_t bias_stride[4];
  const uint8_t* mask;
  int64_t mask_stride[4];
  const sdpa_block_mask_info* block_info;
  uint32_t flags;
} sdpa_params;

/* Bytes of workspace sdpa_forward / sdpa_decode_with_cache need for these params (at least
 * 256: the device status word lives at the start). The workspace must be 256-byte aligned.
 * Returns 0 if the params are invalid. */
SDPA_API size_t sdpa_workspace_size(const sdpa_params* p);

/* Writes the status word at the start of `ws` to SDPA_OK (enqueued on `stream`). Call once on
 * a fresh workspace before the first use; kernels only ever set it to an error. */
SDPA_API sdpa_status sdpa_workspace_init(void* ws, size_t ws_bytes, struct CUstream_st* stream);

/* scaled_dot_product_attention(q, k, v, [bias]; mask, scale, is_causal, q_offset, q_lengths,
 * kv_lengths) into `out` (device, caller-owned, same dtype as q). A query attending to no key
 * gives NaN (section "Fused implementation"). Returns SDPA_OK once the work is enqueued. */
SDPA_API sdpa_status sdpa_forward(const sdpa_params* p, const void* q, const void* k, const void* v,
                         void* out, void* ws, size_t ws_bytes, struct CUstream_st* stream);

/* sdpa_forward that also writes each query row's log-sum-exp, for a gradient that follows
 * (sdpa_backward_lse) without running the forward again. lse: device float
 * [batch][nheads][q_len], natural log, lse_i = log sum_j exp(logit_ij) over the keys row i
 * attends; +inf for a row with no key or past q_lengths. Runs the tcgen05 kernel only:
 * bf16/fp16, qk_head_dim = v_head_dim = 64 or 128, no bias, mask or block_info, no
 * SDPA_FLAG_GENERIC_KERNEL (SDPA_ERR_UNSUPPORTED otherwise). Workspace as sdpa_forward. */
SDPA_API sdpa_status sdpa_forward_lse(const sdpa_params* p, const void* q, const void* k, const void* v,
                                      void* out, float* lse, void* ws, size_t ws_bytes,
                                      struct CUstream_st* stream);

/* Packed sequences (keywords q_segments, kv_segments and maxlen, paragraph "Packed
 * sequences"): nseg sequences stored one after the other along the sequence axis, with no
 * batch axis and no padding.
 *  q_segments   device int32[nseg]: the length of each query sequence.
 *  kv_segments  device int32[nseg]: the length of each key/value sequence, or NULL to reuse
 *               q_segments (the keyword's default).
 *  maxlen       at least every entry of both arrays. The host never reads the lengths: the
 *               work is sized by nseg and maxlen. A segment longer than maxlen is an error,
 *               found on the device. */
typedef struct sdpa_packed_segments {
  int32_t nseg;
  int32_t maxlen;
  const int32_t* q_segments;
  const int32_t* kv_segments;
} sdpa_packed_segments;

/* Workspace bytes sdpa_forward_packed needs (256-byte aligned; 0 if the arguments are
 * invalid). */
SDPA_API size_t sdpa_packed_workspace_size(const sdpa_params* p, const sdpa_packed_segments* seg);

/* scaled_dot_product_attention on packed sequences. The s-th query sequence attends to the
 * s-th key/value sequence only, as batch element s of a padded batch would. is_causal applies
 * within each sequence.
 *  - Layout. q [total_q][nheads][dqk], k [total_kv][nkvheads][dqk], v [total_kv][nkvheads][dv],
 *    out [total_q][nheads][dv]: the page's (head_dim, nheads, total_len). In p: batch = 1,
 *    q_len = total_q, kv_len = total_kv.
 *  - q_offset, q_lengths and kv_lengths, when given, are device int32[nseg], one entry per
 *    sequence. q_lengths[s] and kv_lengths[s] lie in [0, segment length].
 *  - bias, mask and block_info must be NULL (the page supports neither with segments):
 *    SDPA_ERR_INVALID_ARG otherwise.
 *  - Device-side checks. These set SDPA_ERR_DEVICE_CHECK in the status word:
 *      - lengths that are negative;
 *      - lengths above maxlen;
 *      - lengths that do not add up to total_q / total_kv.
 *    Rows are clamped to the arrays whatever the lengths. Rows of a sequence past maxlen are
 *    not computed.
 *  - Kernels. A one-block kernel first turns the lengths into the first row of each sequence
 *    (in the workspace). The attention kernel then runs: tcgen05 for bf16/f16 with
 *    dqk = dv = 64 or 128, the SIMT kernel otherwise. */
SDPA_API sdpa_status sdpa_forward_packed(const sdpa_params* p, const sdpa_packed_segments* seg,
                                         const void* q, const void* k, const void* v, void* out,
                                         void* ws, size_t ws_bytes, struct CUstream_st* stream);

/* scaled_dot_product_attention_with_weights (the entry's "See also": the attention weights
 * too) with fdrop as dropout of probability drop_p (argument fdrop: applied to the weights right
 * after the softmax). The weights are materialized, as the page's materialized implementation
 * does for such calls.
 *  - Arguments are those of sdpa_forward, all supported, bias and mask included.
 *  - weights (device, caller-owned, p->dtype) gets the page's (kv_len, q_len, nheads, batch)
 *    order, row-major [batch][nheads][q_len][kv_len], after the dropout. A row with no attended
 *    key has NaN weights and output. A row past q_lengths has zero weights and output.
 *  - The dropout keeps w_ij, divided by 1 - drop_p, when its draw u >= ceil(drop_p * 2^16),
 *    and otherwise sets it to 0. The weights' row-major positions are taken four at a time:
 *    group g = index / 4 gets r = mix(seed + (g + 1) * 0x9e3779b97f4a7c15), the SplitMix64
 *    generator's output g + 1 from state seed (mix: its finalizer, Steele, Lea and Flood 2014),
 *    and u is the 16-bit field index % 4 of r (lowest first). So a
 *    weight is kept with probability 1 - ceil(drop_p * 2^16) / 2^16, within 2^-16 of
 *    1 - drop_p. drop_p must be in [0, 1), and 0 means no dropout.
 *  - out = weights · v.
 *  - The workspace holds the status word and one float per query row (the row's log-sum-exp):
 *    sdpa_weights_workspace_size(p) bytes.
 *  - Kernels. bf16/fp16 with dqk = dv = 64 or 128, no bias, mask or block_info, kv_len a
 *    multiple of 8 and 16-byte aligned arrays run on the tcgen05 prefill kernel: a statistics
 *    pass (the row log-sum-exp alone), the weights of the key tiles beyond each query tile's
 *    causal / kv_lengths bound (0, or NaN for a row with no key: written by the statistics pass
 *    when no row can be empty, else by a fill kernel), then the weights pass, which recomputes
 *    the logits on the tensor cores, accumulates out from the dropped weights and stores the
 *    weights of the visited tiles through shared memory with TMA. Other
 *    bf16/fp16 calls with dqk = dv = 64 or 128 take mma.sync tiles; a SIMT kernel handles the
 *    rest, or runs when SDPA_FLAG_GENERIC_KERNEL is set. */
SDPA_API size_t sdpa_weights_workspace_size(const sdpa_params* p);
SDPA_API sdpa_status sdpa_forward_with_weights(const sdpa_params* p, double drop_p, uint64_t seed, const void* q,
                                               const void* k, const void* v, void* out, void* weights, void* ws,
                                               size_t ws_bytes, struct CUstream_st* stream);

/* Rotary position embedding of query or key rows, applied after the projections and before
 * attention (the Keras thread "MultiHeadAttention is missing a position_bias call argument"
 * names rotary embeddings but gives no formula). The common form is used:
 *    the pair (c, c + d/2), c < d/2, of row t is rotated by the angle a = positions[t] * base^(-2c/d):
 *    out[c] = x[c] cos a - x[c + d/2] sin a,   out[c + d/2] = x[c + d/2] cos a + x[c] sin a.
 *  - x, out: device arrays of `dtype`, [rows][nheads][d] (a padded batch flattens to
 *    rows = batch * seq_len). out may be x (in place).
 *  - positions: device int32[rows], the position of each row. With a KV cache this is the
 *    absolute position, cache index + t.
 *  - d must be even, at most 8192 (SDPA_ERR_UNSUPPORTED beyond), and base > 0 (10000 is the
 *    usual value). The frequencies and the angle, reduced to [-pi, pi], are taken in double
 *    precision; CUDA's sincosf evaluates the reduced angle and the rotation is in fp32.
 *  - One elementwise kernel; no workspace. */
SDPA_API sdpa_status sdpa_rope(const void* x, void* out, sdpa_dtype dtype, int64_t rows, int32_t nheads, int32_t d,
                               const int32_t* positions, double base, struct CUstream_st* stream);

/* Attention with the rotary position embedding of the queries and keys (the form of sdpa_rope)
 * folded into the call: out = sdpa_forward(p, rope(q, q_positions), rope(k, k_positions), v).
 * The Keras thread "MultiHeadAttention is missing a position_bias call argument" applies the
 * rotary embedding to the query and key right before the attention; here q and k are read
 * as given and not modified.
 *  - q_positions: device int32[batch * q_len], k_positions: device int32[batch * kv_len], the
 *    position of each row (the absolute position; with a cache, cache index + t). base > 0.
 *  - Every argument of sdpa_forward applies to the rotated arrays; qk_head_dim must be even.
 *  - The workspace (sdpa_rope_workspace_size(p) bytes) holds the status word, the rotated keys
 *    (one pass over k: every query tile of a key/value head reads them), a cos / sin table of
 *    the query rows and room for rotated queries.
 *  - Kernels. Where sdpa_forward takes the tcgen05 kernel and there is no bias or mask, a table
 *    kernel computes the query angles' cos / sin and the attention kernel rotates each Q tile
 *    in shared memory after its TMA load, before the first QK^T MMA reads it, so the rotated
 *    queries never go to memory. Otherwise the queries are rotated into the workspace and the
 *    tcgen05 kernel (with a bias or mask) or the SIMT kernel runs.
 *    The rotated values are rounded to the input type, as sdpa_rope's output is. */
SDPA_API size_t sdpa_rope_workspace_size(const sdpa_params* p);
SDPA_API sdpa_status sdpa_forward_rope(const sdpa_params* p, const int32_t* q_positions,
                                       const int32_t* k_positions, double base, const void* q,
                                       const void* k, const void* v, void* out, void* ws,
                                       size_t ws_bytes, struct CUstream_st* stream);

/* Workspace bytes sdpa_backward needs for these params (256-byte aligned; 0 if invalid). */
SDPA_API size_t sdpa_backward_workspace_size(const sdpa_params* p);

/* The gradient of the fused implementation (paragraph "Fused implementation"), with respect
 * to query, key, value and scale, for the loss sum(dout * out). The weights are recomputed
 * from q and k and never materialized.
 *  - Inputs. q, k, v and p are those of the sdpa_forward call that produced `out`. dout has
 *    out's shape. All are device arrays of p->dtype.
 *  - Outputs. dq, dk and dv (device, caller-owned) get the shapes and dtype of q, k and v. A
 *    key/value head sums the contributions of the query heads that share it. dscale is a
 *    device float or NULL.
 *  - Rows that take no part. A query that attends to no key (NaN output) and a query past
 *    q_lengths (zero output) get dq = 0 and add nothing to dk, dv or dscale.
 *  - Arguments. mask, block_info, is_causal, q_offset, q_lengths and kv_lengths are as in
 *    sdpa_forward. A bias is SDPA_ERR_INVALID_ARG: the page's automatic differentiation
 *    takes the materialized implementation for a call with a bias. Head sizes are up to 256.
 *  - Kernels. bf16/fp16 with dqk = dv = 128 and no mask or block_info run on tcgen05: the
 *    forward kernel again for the row log-sum-exp (its output goes to dq, then overwritten),
 *    delta = dout . out, then dk and dv per 128-key tile (resident in TMEM across the query
 *    tiles of the group) and dq and dscale per 128-query tile. dx enters dk and dq as a 16-bit
 *    high part plus the rounded remainder (two MMAs); w enters dv with one rounding. Other
 *    bf16/fp16 calls with dqk = dv = 64 or 128 run two mma.sync tile kernels (dq with the row
 *    log-sum-exp, delta and dscale, then dk and dv per key tile). Other types and sizes, or
 *    SDPA_FLAG_GENERIC_KERNEL, take three SIMT kernels, fp32 throughout. dscale is zeroed
 *    first with cudaMemsetAsync. */
SDPA_API sdpa_status sdpa_backward(const sdpa_params* p, const void* q, const void* k, const void* v,
                                   const void* out, const void* dout, void* dq, void* dk, void* dv,
                                   float* dscale, void* ws, size_t ws_bytes, struct CUstream_st* stream);

/* sdpa_backward given the row log-sum-exp that sdpa_forward_lse wrote for the same call (lse:
 * device float [batch][nheads][q_len], natural log): the tcgen05 gradient then skips its own
 * forward pass. Calls the tcgen05 gradient does not take ignore lse and run as sdpa_backward.
 * Workspace as sdpa_backward. */
SDPA_API sdpa_status sdpa_backward_lse(const sdpa_params* p, const void* q, const void* k, const void* v,
                                       const void* out, const void* dout, const float* lse, void* dq, void* dk,
                                       void* dv, float* dscale, void* ws, size_t ws_bytes,
                                       struct CUstream_st* stream);

/* Decoding with a KV cache (the page's example "decoding with a KV cache"; the Keras issue
 * "MultiHeadAttention is missing a position_bias call argument", cache_update_index):
 * writes k_new/v_new [batch][n_new][nkvheads][d] into k_cache/v_cache
 * [batch][capacity][nkvheads][d] at rows cache_index[b] .. cache_index[b] + n_new - 1, then
 * attends the n_new queries q [batch][n_new][nheads][dqk] with is_causal=:bottom_right and
 * kv_lengths[b] = cache_index[b] + n_new. Here p->q_len = n_new, p->kv_len = capacity,
 * p->causal must be SDPA_CAUSAL_BOTTOM_RIGHT and q_lengths, kv_lengths, bias, mask and
 * block_info must be NULL. cache_index is a device int32[batch]; a value outside
 * [0, capacity - n_new] skips that sequence's cache write and attention, writes NaN to its
 * output rows (so the failure shows in the result) and sets SDPA_ERR_DEVICE_CHECK in the
 * status word. */
SDPA_API sdpa_status sdpa_decode_with_cache(const sdpa_params* p, const void* q, const void* k_new,
                                   const void* v_new, void* k_cache, void* v_cache,
                                   const int32_t* cache_index, void* out, void* ws,
                                   size_t ws_bytes, struct CUstream_st* stream);

/* Decoding with a KV cache for callers that cannot allocate device memory (this entry point
 * has no counterpart in the paper). Some callers cannot call cudaMalloc: plug-ins hosted by a
 * framework that owns every device allocation, or latency-critical decode loops that must never
 * block on, or fail in, the allocator mid-run. They cannot supply the workspace that
 * sdpa_decode_with_cache needs. This call computes the same thing, with the same arguments
 * minus the workspace. Its scratch is a fixed array of SDPA_STATIC_SCRATCH_BYTES inside the
 * library, which every GPU that loads the library holds until the process exits.
 *  - A call whose scratch need (sdpa_workspace_size(p)) exceeds that size is rejected with
 *    SDPA_ERR_WORKSPACE before anything is launched.
 *  - The first call on each device looks up the array's device address with that device
 *    current. Make that first call before any stream capture.
 *  - Every call on a device shares the one array. Calls that overlap on the GPU (other streams,
 *    other host threads) race on it: serialise them.
 *  - Invalid arguments return a status before anything is queued, as for
 *    sdpa_decode_with_cache. A valid call first clears the device status word, which sits in
 *    the array, and then runs the same kernels. An out-of-range cache_index skips that
 *    sequence, writes NaN to its output rows and sets SDPA_ERR_DEVICE_CHECK in that word;
 *    sdpa_read_static_status() returns and clears it.
 *  - 40 MiB holds the partials of a bf16/fp16 decode step of 64 sequences x 8 key/value
 *    heads x capacity 8192 at head_dim 128 (34.1 MB). A call whose sdpa_workspace_size(p)
 *    exceeds it is rejected (first point above).
 *  - Nothing is allocated. No cudaMalloc, cudaFree or allocating library routine is called. */
#define SDPA_STATIC_SCRATCH_BYTES (40u << 20)
SDPA_API sdpa_status sdpa_decode_with_cache_static(const sdpa_params* p, const void* q,
                                                   const void* k_new, const void* v_new,
                                                   void* k_cache, void* v_cache,
                                                   const int32_t* cache_index, void* out,
                                                   struct CUstream_st* stream);

/* The device status word of sdpa_decode_with_cache_static on the current device: synchronises
 * `stream`, returns SDPA_OK or the first device error recorded since the last call that
 * cleared it (every static call clears it when it starts, so this reports the most recent
 * static call), and resets it to SDPA_OK. SDPA_OK if no static call has run on this device.
 * Like the static call it allocates nothing (no counterpart in the paper). */
SDPA_API sdpa_status sdpa_read_static_status(struct CUstream_st* stream);

/* Writes k_new/v_new [batch][n_new][nkvheads][d] of `dtype` into the caches
 * [batch][capacity][nkvheads][d] at rows index[b] + t, t < n_new (index: device
 * int32[batch]). Either cache pair may be NULL to update only the other. An index outside
 * [0, capacity - n_new] skips that sequence and sets SDPA_ERR_DEVICE_CHECK in the status word
 * of `ws` (ws may be NULL, in which case the check is silent). */
SDPA_API sdpa_status cache_update_at_index(void* k_cache, void* v_cache, const void* k_new,
                                  const void* v_new, sdpa_dtype dtype, int32_t d,
                                  int32_t nkvheads, int32_t n_new, int32_t capacity,
                                  int32_t batch, const int32_t* index, void* ws,
                                  struct CUstream_st* stream);

/* Bytes of info buffer build_block_mask_info needs (256-byte aligned). bk must be a multiple
 * of 32. Returns 0 if the sizes are invalid. */
SDPA_API size_t build_block_mask_info_size(int32_t nheads, int32_t q_len, int32_t kv_len, int32_t bq,
                                  int32_t bk);

/* Classifies every bq x bk block of a boolean mask (device uint8, element (key j, query i,
 * head h) at mask[j*mask_stride[0] + i*mask_stride[1] + h*mask_stride[2]]; mask_stride[0]
 * must be 1) as empty, partial or full, packs the bits of the partial blocks and lists the
 * non-empty blocks of every block row (see sdpa_block_mask_info). The result lives in the
 * caller's `info_buf` and is described by *out_info, filled in on the host before return.
 * sdpa_forward uses it when bq = bk = 128. At most 65535 query blocks and 65535 mask heads
 * (SDPA_ERR_INVALID_ARG beyond). Two kernels run on `stream`: one per block, then one that
 * builds the block-row lists. */
SDPA_API sdpa_status build_block_mask_info(const uint8_t* mask, const int64_t mask_stride[3],
                                  int32_t nheads, int32_t q_len, int32_t kv_len, int32_t bq,
                                  int32_t bk, void* info_buf, size_t info_bytes,
                                  sdpa_block_mask_info* out_info, struct CUstream_st* stream);

/* Synchronises `stream`, returns the status word of `ws` (SDPA_OK or the first device error)
 * and resets it to SDPA_OK. For tests and diagnostics; not for the hot path. */
SDPA_API sdpa_status sdpa_read_device_status(void* ws, struct CUstream_st* stream);

/* Message for the last non-OK status returned on this host thread. */
SDPA_API const char* sdpa_last_error(void);

/* Name of the kernel the last sdpa_forward / sdpa_forward_packed / sdpa_forward_lse /
 * sdpa_forward_rope / sdpa_forward_with_weights / sdpa_decode_with_cache / sdpa_backward call on
 * this host thread launched for its attention ("generic_simt", "prefill_tcgen05",
 * "prefill_tcgen05_rope", "decode_splitkv", "weights_tcgen05", "weights_mma", "weights_simt",
 * "backward_tcgen05", "backward_mma", "backward_simt"). */
SDPA_API const char* sdpa_last_kernel(void);

/* 1 in the range-checked build of the library (compiled with SDPA_DEBUG_CHECKS, shipped as
 * libsdpa_debug.so), 0 in the normal one. In the range-checked build every device-side index the
 * kernels take from data (block-row counts and lists, partial-bit addresses, TMA tile
 * coordinates, cache and split indices, output rows) is checked before use; a violation sets
 * SDPA_ERR_DEVICE_CHECK in the status word and the access is skipped (or, for a TMA
 * coordinate, clamped into the array), so a bad input is reported instead of faulting. It is
 * the stand-in for a memory checker and costs speed. */
SDPA_API int sdpa_debug_checks(void);

#ifdef __cplusplus
}
#endif

#endif /* SDPA_H_ */
