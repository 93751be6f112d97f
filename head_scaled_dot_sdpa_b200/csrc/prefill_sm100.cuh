// Tiled online-softmax attention for sm_100a (B200): the fused implementation of
// NNlib.scaled_dot_product_attention (Flux.jl page "Neural Network primitives from NNlib.jl",
// section "Fused implementation": tile by tile, online softmax over key tiles, weights never
// materialised), for fp16/bf16 inputs with qk_head_dim = v_head_dim in {64, 128}.
//
// Work unit: two 128-query tiles A and B that read the same key/value head of the same batch
// element: two query heads of one GQA group (same query tile), or, without GQA, two adjacent
// query tiles of one head. Persistent CTAs (one per SM) walk the units, longest causal rows
// first. The key tiles a unit visits are the union of the two tiles' lists (the causal /
// kv_lengths prefix, or the non-empty blocks of a block-sparse mask), each loaded once.
//
// Warp roles (384 threads):
//   warp 8      TMA producer: Q_A, Q_B, then K_u ahead of V_{u-1} (and the bias tiles of the
//               shared-memory bias variant) through 128B-swizzled rings; it also takes the units
//               from the counter and prefetches their Q tiles into L2;
//   warps 9, 11 MMA issuers of tile A and tile B (warp 9 owns the TMEM; warp 10 idle;
//               warpgroup 2 gives its registers to the softmax warpgroups with setmaxnreg).
//               Per key tile u each issues O_X += P_X(u-1) V(u-1); S_X(u) = Q_X K(u)^T (S:
//               both operands in shared memory; PV: P read from TMEM; the in-order tcgen05
//               pipeline lets S_X(u) reuse the columns PV_X(u-1) just read). A turn order
//               between the two warps keeps the issue order A, B, A, B, so the tensor pipe
//               works on one tile while the other tile's softmax runs; each waits for V, K
//               and P before its turn, so the turn is the last wait before its MMAs;
//   warps 0-3   softmax of tile A, warps 4-7 softmax of tile B: one thread per query row
//               (= TMEM lane). tcgen05.ld of the S row; masks (causal / q_offset / kv_lengths
//               as one prefix bound per row, boolean mask bytes or partial-block bits); optional
//               bias; row max; P = 2^(s*scale*log2e - m) written back into the S columns as
//               16-bit pairs (tcgen05.st). The running max m only moves when the row max passes
//               it by more than 2^8, so every exponential stays <= 256; O and the row sum are
//               then rescaled in TMEM (the commit that signalled S(u) also covers PV(u-1), so O
//               is at rest). Epilogue: O / l, NaN for rows with no key, 0 past q_lengths.
//
// Every mbarrier wait is bounded (P.wait_timeout_ns); on a timeout the CTA records
// SDPA_ERR_TIMEOUT in the status word, every role unwinds and the TMEM is released.
#pragma once

#include <cuda.h>

#include <atomic>
#include <type_traits>

#include "device_common.cuh"
#include "sm100_primitives.cuh"

namespace sdpa {
namespace prefill {

using namespace sm100;

constexpr int kBlockM = 128;
constexpr int kBlockN = 128;
// With head_dim 64, P is handed to the MMA warp in two parts: the first kEarlyKeys keys as
// soon as they are written (their PV steps start while the softmax finishes the rest), then the
// remainder. (With head_dim 128 the split was measured 1-2% slower and P goes in one part.)
constexpr int kEarlyKeys = 96;
// With head_dim 64 and no bias the forward keeps P in TMEM columns of its own (384 + 64 *
// stream: S and O take 384 of the 512): the next S is issued as soon as the softmax has read S,
// and PV follows P, so the MMAs overlap the softmax instead of following it. (Measured: 3.5 %
// faster without a bias, 8 % slower with the bias tiles, which keep P over S with the two-part
// hand-over, as do the other modes.)
template <int D, int kMode, int kBias>
constexpr bool kSepP = D == 64 && (kMode == 0 || kMode == 1) && kBias == 0;
template <int D, int kMode, int kBias>
constexpr bool kSplitP = D == 64 && !kSepP<D, kMode, kBias>;
// With head_dim 128 the forward writes O through a shared-memory staging tile and TMA stores
// (one per 64-dim half), so that the stores are whole lines and leave the softmax warps at once.
template <int D, int kMode>
constexpr bool kOStage = D == 128 && (kMode == 0 || kMode == 1);
// The weights pass stores its weight tiles through the same staging tiles (each softmax warp its
// 32 rows, one 64-key half at a time), with either head_dim.
template <int D, int kMode>
constexpr bool kStageSmem = kOStage<D, kMode> || kMode == 2;
constexpr int kThreads = 384;  // 3 warpgroups: softmax A, softmax B, producer + MMA (+2 idle)
// Register split (setmaxnreg): the two softmax warpgroups grow to kSoftmaxRegs, the last one
// shrinks to kOtherRegs. 2*128*216 + 128*72 = 64512 = 384 * 168, the launch's registers; the
// host refuses to launch unless the kernel was compiled with >= kLaunchRegs per thread.
constexpr int kSoftmaxRegs = 216;
constexpr int kOtherRegs = 72;
constexpr int kLaunchRegs = 168;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kRegionBytes = 128 * 128;    // 128 rows x 128 bytes (64 16-bit columns)
constexpr int kNone = 1 << 30;
constexpr int kUnitSlots = 4;        // ring of unit indices handed from the producer to the others
constexpr int kUnitInfoBytes = 128;  // per ring slot: the unit's decomposition (struct Unit)
constexpr int kUnitConsumers = 10;   // the two MMA warps and the 8 softmax warps
constexpr int kMmaWarpA = 9, kMmaWarpB = 11;  // MMA issuers of tile A and tile B
constexpr int kSchedWord = 16;       // int offset in the status area of the unit counter (+1: done)

// bias / mask variants compiled into the kernel
// kBiasTile: a 16-bit bias brought into shared memory by TMA, one 128 x 128 tile per query tile
// and key tile (head_dim 64, where the shared memory holds it); the others read global memory.
enum { kBiasNone = 0, kBiasSame = 1, kBiasF32 = 2, kBiasTile = 3 };
enum { kMaskNone = 0, kMaskDense = 1, kMaskBits = 2 };
// kModeForward: the attention output. kModeAux: the same, and (no bias or mask) each row's
// log-sum-exp when P.lse is set and the rotary embedding of the Q tiles when P.q_rope is set.
// kModeWeights: scaled_dot_product_attention_with_weights given that log-sum-exp: the exact
// weights 2^(x - lse) of the visited key tiles, dropped out and stored, and out = sum w' v.
// kModeStats: each row's log-sum-exp alone (P.lse; no bias or mask), for the weights pass that
// follows: no V tiles, no PV, no output; the next S is issued as soon as the softmax has read
// the current one. (The plain forward carries none of the extra code.)
enum { kModeForward = 0, kModeAux = 1, kModeWeights = 2, kModeStats = 3 };

// Shared-memory plan: the Q tiles of the two query tiles, the K and V rings, and with bias
// tiles (kBT, head_dim 64) one bias tile per query tile. (A third Q slot, so that the next
// unit's first Q tile loads a whole unit ahead, and two bias tiles in flight per query tile
// were measured on B200 and were 1-2 % slower; the slot counts stay parameters.)
template <int D, bool kBT = false>
struct Cfg {
  static constexpr int kRegions = D / 64;
  static constexpr int kTileBytes = kRegions * kRegionBytes;
  static constexpr int kKStages = D == 128 ? 2 : 4;
  static constexpr int kVStages = D == 128 ? 2 : 4;
  static constexpr int kBiasTileBytes = 128 * 128 * 2;
  static constexpr int kBiasSlots = 1;  // per query tile
  // Q tiles: a ring shared by the two query tiles of the units, in the order A, B, A, B, ...
  static constexpr int kQSlots = 2;
  static constexpr int kBiasBytes = kBT ? 2 * kBiasSlots * kBiasTileBytes : 0;
  // O staging (kOStage): one 128-row x 64-dim tile per query tile
  static constexpr int kOStageBytes = 2 * 128 * 128;
  static constexpr int kBarriers =
      3 * kQSlots + 2 * kKStages + 2 * kVStages + 2 * 4 + 2 * 2 * kBiasSlots + 1 + 2 * kUnitSlots + 8;
  // tiles (+ the bias tiles), barriers, unit ring, TMEM address, abort flag, and slack to align
  // the base to 1024 bytes
  static constexpr int smem_bytes(bool ostage = false) {
    return (kQSlots + kKStages + kVStages) * kTileBytes + kBiasBytes + (ostage ? kOStageBytes : 0) + kBarriers * 8 +
           64 + kUnitSlots * kUnitInfoBytes + 16 + 1024;
  }
};
static_assert(Cfg<64, true>::smem_bytes() <= 227 * 1024, "bias tiles fit for head_dim 64");
static_assert(Cfg<128>::smem_bytes(true) <= 227 * 1024 && Cfg<64>::smem_bytes() <= 227 * 1024, "tiles fit");

struct TensorMaps {
  CUtensorMap q, k, v, bias;  // bias: (keys, queries, heads, batch), used by kBiasTile only
  CUtensorMap o;              // out, as q (the staged epilogue's stores)
  CUtensorMap w;              // weights (keys, queries, heads, batch), box 64 x 128: the zero fill
  CUtensorMap w_warp;         // the same, box 64 keys x 32 rows: one warp's staged weights
};

// One query tile of a unit.
struct QTile {
  int h, qt, i0, n;      // n = number of key tiles it visits
  const uint32_t* list;  // block list (kb | class << 30), or null for the prefix 0..n-1
  __device__ __forceinline__ int kb(int j) const { return list ? (int)(list[j] & 0x3FFFFFFFu) : j; }
  __device__ __forceinline__ int next(int j) const { return j < n ? kb(j) : kNone; }
};

struct Unit {
  int b, kvh;
  int q_len, kv_len, offset;
  int q_rows;       // rows of the sequence in q / out; rows past it are another sequence's
  int tq, tk, tb;   // TMA coordinates: first query row, first key row, batch index
  long long o0;     // first row of the sequence in out viewed as (rows, heads, head_dim)
  QTile t[2];
};
static_assert(sizeof(Unit) <= kUnitInfoBytes, "unit ring slot");

__device__ __forceinline__ QTile make_qtile(const Problem& P, const BatchInfo& bi, int h, int qt, bool present) {
  QTile x;
  x.h = h;
  x.qt = qt;
  x.i0 = qt * kBlockM;
  x.list = nullptr;
  x.n = 0;
  if (!present || bi.skip || x.i0 >= bi.q_len) return x;
  int n_lim = (bi.kv_len + kBlockN - 1) / kBlockN;
  if (P.causal != SDPA_CAUSAL_NONE) {
    const long long last_row = min(x.i0 + kBlockM - 1, bi.q_len - 1);
    const long long last_key = (long long)bi.offset + last_row;
    n_lim = last_key < 0 ? 0 : (int)min((long long)n_lim, last_key / kBlockN + 1);
  }
  if (P.bcls) {
    const int hm = P.bi_nheads == 1 ? 0 : h;
    const long long row = (long long)hm * P.bi_nqb + qt;
    // range-checked build: the block row must exist and its count fit the row
    if (!SDPA_CHECKED(P.status, hm < P.bi_nheads && qt < P.bi_nqb)) return x;
    x.list = P.brow_list + row * P.bi_nkb;
    int cnt = P.brow_count[row];
    if (!SDPA_CHECKED(P.status, cnt >= 0 && cnt <= P.bi_nkb)) cnt = cnt < 0 ? 0 : P.bi_nkb;
    int n = 0;
    while (n < cnt && (int)(x.list[n] & 0x3FFFFFFFu) < n_lim) ++n;
    x.n = n;
  } else {
    x.n = n_lim;
  }
  return x;
}

// Units: with GQA, (query tile, batch, kv head, head pair); without, (tile pair, batch, head).
// Enumerated longest causal rows first.
__host__ __device__ __forceinline__ int units_per_level(const Problem& P) {
  return P.group >= 2 ? P.B * P.Hkv * ((P.group + 1) / 2) : P.B * P.H;
}
__host__ __device__ __forceinline__ int n_levels(const Problem& P) {
  const int nqt = (P.Lq + kBlockM - 1) / kBlockM;
  return P.group >= 2 ? nqt : (nqt + 1) / 2;
}

__device__ __forceinline__ Unit make_unit(const Problem& P, int u) {
  Unit w;
  const int per = units_per_level(P);
  const int level = n_levels(P) - 1 - u / per;
  const int rem = u % per;
  const int nqt = (P.Lq + kBlockM - 1) / kBlockM;
  int hA, hB, qA, qB;
  bool haveB;
  if (P.group >= 2) {
    const int pairs = (P.group + 1) / 2;
    w.b = rem / (P.Hkv * pairs);
    const int r2 = rem % (P.Hkv * pairs);
    w.kvh = r2 / pairs;
    const int pr = r2 % pairs;
    hA = w.kvh * P.group + 2 * pr;
    hB = hA + 1;
    haveB = 2 * pr + 1 < P.group;
    qA = qB = level;
  } else {
    w.b = rem / P.H;
    hA = hB = rem % P.H;
    w.kvh = hA;
    qA = 2 * level;
    qB = qA + 1;
    haveB = qB < nqt;
  }
  const BatchInfo bi = resolve_batch(P, w.b);
  w.q_len = bi.q_len;
  w.kv_len = bi.kv_len;
  w.offset = bi.offset;
  w.q_rows = bi.q_rows;
  w.o0 = bi.q0;
  // a padded batch is a 4-d map indexed by batch; packed sequences are one batch of all rows,
  // each sequence starting at its own row
  const bool packed = P.q_start != nullptr;
  w.tq = packed ? (int)bi.q0 : 0;
  w.tk = packed ? (int)bi.k0 : 0;
  w.tb = packed ? 0 : w.b;
  w.t[0] = make_qtile(P, bi, hA, qA, true);
  w.t[1] = make_qtile(P, bi, hB, qB, haveB);
  if (!haveB) w.t[1].i0 = kNone;  // marks "no tile B"
  return w;
}

template <typename BT>
__device__ __forceinline__ void load8(const BT* p, float (&f)[8]) {
  if constexpr (std::is_same<BT, float>::value) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  } else {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      BT lo, hi;
      const uint16_t l16 = (uint16_t)(w[k] & 0xFFFFu), h16 = (uint16_t)(w[k] >> 16);
      lo = *reinterpret_cast<const BT*>(&l16);
      hi = *reinterpret_cast<const BT*>(&h16);
      f[2 * k] = to_f32(lo);
      f[2 * k + 1] = to_f32(hi);
    }
  }
}

// O (D fp32 columns of this thread's TMEM lane) *= a. Rare (the running max moved by more
// than 2^8), so it is kept out of line: its code and registers stay off the softmax loop.
template <int D>
__device__ __noinline__ void rescale_o(uint32_t taddr, float a) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tmem_ld32(taddr + c * 32, o);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a);
    tmem_st32(taddr + c * 32, o);
  }
  tmem_wait_st();
}

// Rotary embedding of row r of a Q tile in shared memory (128-byte swizzle: logical 16-byte
// chunk x of row r is stored at chunk x ^ (r % 8)): the pair (c, c + D/2) rotated by the angle
// whose (cos, sin) fp16 pair is table[c]. Inlined: it runs where the softmax's score registers
// are not live (an out-of-line call saved and restored them around every rotation).
template <typename T, int D>
__device__ __forceinline__ void rotate_q_row(uint8_t* tile, int r, const uint32_t* table) {
  constexpr int kHalf = D / 2, kPairChunks = kHalf / 8;
  const uint4* trow = reinterpret_cast<const uint4*>(table);
  uint4 tab[2 * kPairChunks];
#pragma unroll
  for (int z = 0; z < 2 * kPairChunks; ++z) tab[z] = trow[z];
#pragma unroll
  for (int x = 0; x < kPairChunks; ++x) {
    uint8_t* lo = tile + r * 128 + ((x ^ (r & 7)) << 4);
    uint8_t* hi = D == 128 ? lo + kRegionBytes : tile + r * 128 + (((x + 4) ^ (r & 7)) << 4);
    uint4 a = *reinterpret_cast<uint4*>(lo), b = *reinterpret_cast<uint4*>(hi);
    uint32_t* pa = reinterpret_cast<uint32_t*>(&a);
    uint32_t* pb = reinterpret_cast<uint32_t*>(&b);
    const uint32_t* cs = reinterpret_cast<const uint32_t*>(&tab[2 * x]);  // 8 (cos, sin) pairs
#pragma unroll
    for (int z = 0; z < 4; ++z) {
      float y0[2], y1[2];
#pragma unroll
      for (int y = 0; y < 2; ++y) {
        const uint16_t la = (uint16_t)(pa[z] >> (16 * y)), lb = (uint16_t)(pb[z] >> (16 * y));
        const float x0 = to_f32(*reinterpret_cast<const T*>(&la));
        const float x1 = to_f32(*reinterpret_cast<const T*>(&lb));
        const __half2 t2 = *reinterpret_cast<const __half2*>(&cs[2 * z + y]);
        const float cv = __low2float(t2), sv = __high2float(t2);
        y0[y] = x0 * cv - x1 * sv;
        y1[y] = x1 * cv + x0 * sv;
      }
      pa[z] = std::is_same<T, __half>::value ? pack_f16x2(y0[0], y0[1]) : pack_bf16x2(y0[0], y0[1]);
      pb[z] = std::is_same<T, __half>::value ? pack_f16x2(y1[0], y1[1]) : pack_bf16x2(y1[0], y1[1]);
    }
    *reinterpret_cast<uint4*>(lo) = a;
    *reinterpret_cast<uint4*>(hi) = b;
  }
}

template <typename T, int D, int kBias, int kMask, int kMode = kModeForward>
__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ TensorMaps maps, const Problem P, T* __restrict__ out, int n_units) {
  using C = Cfg<D, kBias == kBiasTile>;
  using BT = typename std::conditional<kBias == kBiasF32, float, T>::type;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem;  // [kQSlots] tiles
  uint8_t* k_smem = q_smem + C::kQSlots * C::kTileBytes;
  uint8_t* v_smem = k_smem + C::kKStages * C::kTileBytes;
  uint8_t* b_smem = v_smem + C::kVStages * C::kTileBytes;  // [2][kBiasSlots] bias tiles (kBiasTile)
  uint8_t* o_stage = b_smem + C::kBiasBytes;  // [2] staging tiles of O or of the weights (kStageSmem)
  uint64_t* bars = reinterpret_cast<uint64_t*>(o_stage + (kStageSmem<D, kMode> ? C::kOStageBytes : 0));
  uint64_t* q_full = bars;                  // [kQSlots]
  uint64_t* q_empty = q_full + C::kQSlots;  // [kQSlots]
  uint64_t* k_full = q_empty + C::kQSlots;  // [KS]
  uint64_t* k_empty = k_full + C::kKStages;
  uint64_t* v_full = k_empty + C::kKStages; // [VS]
  uint64_t* v_empty = v_full + C::kVStages;
  uint64_t* s_full = v_empty + C::kVStages; // [2]
  uint64_t* p_full = s_full + 2;            // [2]
  uint64_t* o_ready = p_full + 2;           // [2]
  uint64_t* o_free = o_ready + 2;           // [2]
  uint64_t* b_full = o_free + 2;            // [2][kBiasSlots] bias tile of the stream loaded
  uint64_t* b_empty = b_full + 2 * C::kBiasSlots;  // [2][kBiasSlots] bias tile read by the stream's softmax
  uint64_t* drain = b_empty + 2 * C::kBiasSlots;
  uint64_t* q_rot = drain + 1;                   // [kQSlots] Q tile rotated (P.q_rope)
  uint64_t* unit_full = q_rot + C::kQSlots;      // [kUnitSlots]
  uint64_t* unit_empty = unit_full + kUnitSlots; // [kUnitSlots]
  // [2] the first kEarlyKeys keys of P written (kSepP: S read into the softmax's registers)
  uint64_t* p_early = unit_empty + kUnitSlots;
  uint64_t* p_free = p_early + 2;  // [2] kSepP: the PV of the stream's last P has completed
  uint64_t* stage_free = p_free + 2;      // [2] kOStage: the stream's staging tile may be rewritten
  uint64_t* stage_full = stage_free + 2;  // [2] kOStage: the staging tile is written
  int* unit_ring = reinterpret_cast<int*>(stage_full + 2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(unit_ring + kUnitSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // MMA groups issued so far by the MMA warp of tile A / tile B (the turn order below)
  volatile uint32_t* issued = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);  // [2]
  // the decomposition of the unit in each ring slot, written by the producer with the index
  Unit* unit_info = reinterpret_cast<Unit*>((reinterpret_cast<uintptr_t>(tmem_slot + 4) + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint64_t tmo = P.wait_timeout_ns;

  if (threadIdx.x == 0) {
    for (int x = 0; x < C::kQSlots; ++x) {
      mbar_init(&q_full[x], 1);
      mbar_init(&q_empty[x], 1);
      mbar_init(&q_rot[x], 4);  // one arrive per softmax warp of the tile
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);  // one arrive per softmax warp
      mbar_init(&p_early[s], 4);
      mbar_init(&p_free[s], 1);
      mbar_init(&stage_free[s], 1);  // the stream's leader thread, once the last store has read it
      mbar_init(&stage_full[s], 4);  // one arrive per softmax warp
      mbar_init(&o_ready[s], 1);
      mbar_init(&o_free[s], 4);
    }
    for (int x = 0; x < 2 * C::kBiasSlots; ++x) {
      mbar_init(&b_full[x], 1);
      mbar_init(&b_empty[x], 4);  // one arrive per softmax warp
    }
    // a K / V slot is released by both MMA warps
    for (int s = 0; s < C::kKStages; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 2); }
    for (int s = 0; s < C::kVStages; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 2); }
    mbar_init(drain, 2);
    for (int k = 0; k < kUnitSlots; ++k) {
      mbar_init(&unit_full[k], 1);
      mbar_init(&unit_empty[k], kUnitConsumers);
    }
    *abort_flag = 0;
    issued[0] = 0;
    issued[1] = 0;
    fence_barrier_init();
  }
  if constexpr (kMode == kModeStats) {
    // the zero tile of the weights fill: 64 keys x 128 rows, in the V ring (no V here)
    if (P.stats_fill) {
      for (int x = threadIdx.x; x < 128 * 128 / 16; x += blockDim.x)
        reinterpret_cast<uint4*>(v_smem)[x] = make_uint4(0u, 0u, 0u, 0u);
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    }
  }
  if (warp == kMmaWarpA) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
    if (kBias == kBiasTile) prefetch_tmap(&maps.bias);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&]() {
    *abort_flag = 1;
    report(P.status, SDPA_ERR_TIMEOUT);
  };
  // every lane of a warp takes the same branch; a timeout seen by any lane stops the warp
  // (A phase that has already completed is the common case: one try_wait and a vote settle it
  // without the divergent polling loop, whose reconvergence costs tens of cycles.)
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    const bool ok = mbar_wait(bar, parity, tmo, abort_flag);
    if (__all_sync(0xffffffffu, ok)) return true;
    fail();
    return false;
  };
  const bool elected = lane == 0;
  // Dynamic scheduling: the producer takes units from a counter in the workspace (units are
  // numbered longest causal rows first) and hands them to the other roles through a small ring.
  unsigned int* sched = reinterpret_cast<unsigned int*>(P.status) + kSchedWord;
  // consumers: the k-th unit of this CTA and its decomposition (copied before the slot is released)
  auto next_unit = [&](uint32_t k, int& u, Unit& w) -> bool {
    const int slot = k % kUnitSlots;
    if (!wait_all(&unit_full[slot], (k / kUnitSlots) & 1)) return false;
    u = *reinterpret_cast<volatile int*>(&unit_ring[slot]);
    if (u < n_units) w = unit_info[slot];
    __syncwarp();
    if (elected) mbar_arrive(&unit_empty[slot]);
    return true;
  };

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kOtherRegs));
  }
  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    [&] {
      uint32_t g = 0;            // key tiles loaded so far (ring position)
      uint32_t qi = 0;           // Q tiles loaded so far (ring position)
      uint32_t bc[2] = {0, 0};   // bias tiles loaded per stream
      // extents of the tensor maps (packed sequences: one batch of all rows)
      const bool packed_rows = P.q_start != nullptr;
      const int q_rows_all = packed_rows ? P.Lq_total : P.Lq, kv_rows_all = packed_rows ? P.Lk_total : P.Lk;
      const int n_batch = packed_rows ? 1 : P.B;
      (void)q_rows_all; (void)kv_rows_all; (void)n_batch;
      // self-test: wait for a phase no one completes (the consumers' first release of slot 0)
      if (P.selftest_stall && !wait_all(&unit_empty[0], 0)) return;
      for (uint32_t k = 0;; ++k) {
        const int slot = k % kUnitSlots;
        if (!wait_all(&unit_empty[slot], ((k / kUnitSlots) & 1) ^ 1)) return;
        int u = 0;
        if (elected) {
          // the unit's decomposition is computed once, here, and handed over with its index:
          // its integer divisions stay off the MMA and softmax warps' path between units
          u = (int)atomicAdd(sched, 1u);
          if (u > n_units) u = n_units;
          if (u < n_units) unit_info[slot] = make_unit(P, u);
          unit_ring[slot] = u;
          mbar_arrive(&unit_full[slot]);
        }
        u = __shfl_sync(0xffffffffu, u, 0);
        if (u >= n_units) break;
        __syncwarp();
        const Unit w = unit_info[slot];
        if (w.t[0].n == 0 && w.t[1].n == 0) continue;
        // The unit's Q tiles come from DRAM (each is read once); their slots free only when
        // the previous unit's last S completes, so they are first brought into L2 now, about
        // two key tiles before that.
        if (elected) {
#pragma unroll
          for (int s = 0; s < 2; ++s)
            if (w.t[s].n > 0)
              for (int r = 0; r < C::kRegions; ++r) tma_prefetch_l2_4d(&maps.q, r * 64, w.t[s].h, w.tq + w.t[s].i0, w.tb);
        }
        __syncwarp();
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          if (w.t[s].n == 0) continue;
          const int qs = (int)(qi % C::kQSlots);
          if (!wait_all(&q_empty[qs], ((qi / C::kQSlots) & 1) ^ 1)) return;
          if (elected) {
            int qh = w.t[s].h, qrow = w.tq + w.t[s].i0, qb = w.tb;
            // range-checked build: a tile outside q is reported and read at the origin instead
            if (!SDPA_CHECKED(P.status, qh < P.H && qrow < q_rows_all && qb < n_batch)) qh = qrow = qb = 0;
            mbar_arrive_expect_tx(&q_full[qs], C::kTileBytes);
            for (int r = 0; r < C::kRegions; ++r)
              tma_load_4d(q_smem + qs * C::kTileBytes + r * kRegionBytes, &maps.q, &q_full[qs], r * 64,
                          qh, qrow, qb);
          }
          ++qi;
        }
        // union of the two tiles' key lists; K_u is loaded ahead of V_{u-1}
        int ja = 0, jb = 0, prev_kb = -1;
        for (;;) {
          const int na = w.t[0].next(ja), nb = w.t[1].next(jb);
          const int kb = min(na, nb);
          if (kb != kNone) {
            const uint32_t x = g;
            const int ks = x % C::kKStages;
            if (!wait_all(&k_empty[ks], ((x / C::kKStages) & 1) ^ 1)) return;
            if (elected) {
              int kh = w.kvh, krow = w.tk + kb * kBlockN, kbt = w.tb;
              if (!SDPA_CHECKED(P.status, kh < P.Hkv && krow < kv_rows_all && kbt < n_batch)) kh = krow = kbt = 0;
              mbar_arrive_expect_tx(&k_full[ks], C::kTileBytes);
              for (int r = 0; r < C::kRegions; ++r)
                tma_load_4d(k_smem + ks * C::kTileBytes + r * kRegionBytes, &maps.k, &k_full[ks], r * 64,
                            kh, krow, kbt);
            }
          }
          if (kMode != kModeStats && prev_kb >= 0) {
            const uint32_t x = g - 1;
            const int vs = x % C::kVStages;
            if (!wait_all(&v_empty[vs], ((x / C::kVStages) & 1) ^ 1)) return;
            if (elected) {
              int vh = w.kvh, vrow = w.tk + prev_kb * kBlockN, vbt = w.tb;
              if (!SDPA_CHECKED(P.status, vh < P.Hkv && vrow < kv_rows_all && vbt < n_batch)) vh = vrow = vbt = 0;
              mbar_arrive_expect_tx(&v_full[vs], C::kTileBytes);
              for (int r = 0; r < C::kRegions; ++r)
                tma_load_4d(v_smem + vs * C::kTileBytes + r * kRegionBytes, &maps.v, &v_full[vs], r * 64,
                            vh, vrow, vbt);
            }
          }
          if constexpr (kBias == kBiasTile) {
            // the bias tile (queries of the stream's tile x keys of kb) into the stream's next
            // slot, once the stream's softmax has read the tile that slot held; broadcast
            // dimensions use coordinate 0. The stream's following bias tile is brought into L2
            // now, one key tile ahead of its own load.
            if (kb != kNone) {
#pragma unroll
              for (int s = 0; s < 2; ++s) {
                if ((s == 0 ? na : nb) != kb) continue;
                const int slot = (int)(bc[s] % C::kBiasSlots);
                uint64_t* full = &b_full[s * C::kBiasSlots + slot];
                if (!wait_all(&b_empty[s * C::kBiasSlots + slot], ((bc[s] / C::kBiasSlots) & 1) ^ 1)) return;
                if (elected) {
                  int hb = P.bs[2] != 0 ? w.t[s].h : 0, bb = P.bs[3] != 0 ? w.b : 0;
                  int bkey = kb * kBlockN, bq = w.t[s].i0;
                  if (!SDPA_CHECKED(P.status, bkey < P.Lk && bq < P.Lq && hb < P.H && bb < P.B)) hb = bb = bkey = bq = 0;
                  mbar_arrive_expect_tx(full, C::kBiasTileBytes);
                  uint8_t* dst = b_smem + (s * C::kBiasSlots + slot) * C::kBiasTileBytes;
                  for (int r = 0; r < 2; ++r)
                    tma_load_4d(dst + r * kRegionBytes, &maps.bias, full, bkey + r * 64, bq, hb, bb);
                  const int kn = w.t[s].next((s == 0 ? ja : jb) + 1);
                  if (kn != kNone && kn * kBlockN < P.Lk)
                    for (int r = 0; r < 2; ++r) tma_prefetch_l2_4d(&maps.bias, kn * kBlockN + r * 64, bq, hb, bb);
                }
                ++bc[s];
              }
            }
          }
          __syncwarp();
          if (kb == kNone) break;
          if (na == kb) ++ja;
          if (nb == kb) ++jb;
          prev_kb = kb;
          ++g;
        }
      }
    }();
  } else if (warp == kMmaWarpA || warp == kMmaWarpB) {
    // ------------------------------------------------------------------ MMA issuers
    // One warp per query tile, so that each tile's PV and next S are issued as soon as its
    // own P is ready, whatever the other tile is doing. Both walk the union of the two key
    // lists in the same order; each releases every K / V slot once: by a commit after its
    // last MMA on the slot, or, for a key tile it does not visit, by an arrive once the slot
    // holds that tile (so the arrive always counts toward the slot's current phase).
    [&] {
      const int s = warp == kMmaWarpA ? 0 : 1;
      constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
      constexpr uint32_t idesc_qk = instr_desc_f16(kBf16, false, false, kBlockM, kBlockN);
      constexpr uint32_t idesc_pv = instr_desc_f16(kBf16, false, true, kBlockM, D);
      const uint32_t q_base = smem_addr(q_smem);
      const uint32_t k_base = smem_addr(k_smem), v_base = smem_addr(v_smem);
      const uint32_t s_tmem = tmem + s * 128, o_tmem = tmem + 256 + s * D;
      // Turn order. A tile's MMAs come in groups: S(0); PV(j-1) + S(j); the last PV. Group k
      // of tile A follows group k-1 of tile B, and group k of B follows group k of A, as a
      // single issuer would order them, so the two softmaxes stay half a period apart.
      // Only used when one key list is a prefix of the other (no block list): then neither
      // warp can wait on a K / V slot the other has yet to release.
      const bool turns = P.bcls == nullptr;
      uint32_t base_o = 0;        // groups the other tile issued before this unit
      uint32_t mine = 0;          // groups this warp has issued in total
      auto turn_wait = [&](uint32_t target) -> bool {
        if (!turns || issued[s ^ 1] >= target) return true;
        const uint64_t t0 = global_timer_ns();
        for (uint32_t n = 1;; ++n) {
          if (issued[s ^ 1] >= target) return true;
          if ((n & 255u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > tmo) {
              fail();
              return false;
            }
          }
        }
      };
      // the elected lane publishes a group as soon as its last MMA is issued (before the
      // commits): the other warp may then queue its own group behind it
      auto publish = [&]() { issued[s] = mine + 1; };
      uint32_t g = 0, sc = 0, qi = 0, oc = 0;  // qi: Q tiles of both streams so far (ring position)
      for (uint32_t kq = 0;; ++kq) {
        int u;
        Unit w;
        if (!next_unit(kq, u, w)) return;
        if (u >= n_units) break;
        if (w.t[0].n == 0 && w.t[1].n == 0) continue;
        // (selects on scalars only: an index that depends on the warp would put the unit in
        // local memory)
        const int my_n = s == 0 ? w.t[0].n : w.t[1].n;
        const int n_o = s == 0 ? w.t[1].n : w.t[0].n;
        // groups per tile: S(0); PV(j-1) + S(j); the last PV (statistics only: one per S)
        const uint32_t groups_o =
            n_o > 0 ? (uint32_t)n_o + ((kMode == kModeStats || kSepP<D, kMode, kBias>) ? 0u : 1u) : 0u;
        // group k of this tile may be issued once the other tile has issued `before(k)` groups
        auto before = [&](uint32_t k) -> uint32_t { return base_o + min(s == 0 ? k : k + 1, groups_o); };
        // this tile's place in the Q ring: tile A, then tile B, of every unit with keys
        const uint32_t my_qi = qi + ((s == 1 && w.t[0].n > 0) ? 1u : 0u);
        qi += (w.t[0].n > 0 ? 1u : 0u) + (w.t[1].n > 0 ? 1u : 0u);
        const int qslot = (int)(my_qi % C::kQSlots);
        const uint32_t qtile = q_base + qslot * C::kTileBytes;
        if (my_n > 0) {
          // the Q tile loaded (and, with the rotary embedding, rotated in place)
          if (!wait_all((kMode == kModeAux && P.q_rope) ? &q_rot[qslot] : &q_full[qslot], (my_qi / C::kQSlots) & 1))
            return;
        }
        // V(x) loaded and, for the unit's first PV, O free: waited for ahead of the turn, so
        // that they are off the path from "P ready" to the MMA issue
        // (and P(x) written: usually long before the turn comes, so that the turn is the last
        // wait before the MMAs)
        auto pv_ready = [&](uint32_t x, bool first) -> bool {
          const int vs = x % C::kVStages;
          if (!wait_all(&v_full[vs], (x / C::kVStages) & 1)) return false;
          if (first && !wait_all(&o_free[s], (oc & 1) ^ 1)) return false;
          return wait_all(kSplitP<D, kMode, kBias> ? &p_early[s] : &p_full[s], (sc - 1) & 1);
        };
        // O += P(x) V(x) for this tile's key tile at ring position x (after pv_ready): the steps
        // over the first kEarlyKeys keys, then, once the rest of P is written, the others (they
        // queue behind the first ones on a tensor pipe that is still busy); `last`: the group
        // ends here and is published
        auto pv = [&](uint32_t x, bool first, bool last) -> bool {
          const int vs = x % C::kVStages;
          const uint32_t vtile = v_base + vs * C::kTileBytes;
          // B = V (keys x dims, dims contiguous): MN-major; 64-dim regions kRegionBytes apart
          // (LBO), 8-key groups 1024 bytes apart (SBO); 16 keys per step.
          auto steps = [&](int k0, int k1) {
#pragma unroll
            for (int kk = k0; kk < k1; ++kk) {
              const uint64_t bdesc = smem_desc_sw128(vtile + kk * 16 * 128, kRegionBytes, 1024);
              mma_ts(o_tmem, s_tmem + kk * 8, bdesc, idesc_pv, (first && kk == 0) ? 0u : 1u);
            }
          };
          tc_fence_after();
          if constexpr (!kSplitP<D, kMode, kBias>) {
            if (elected) {
              steps(0, kBlockN / 16);
              if (last) publish();
              mma_commit(&v_empty[vs]);
            }
            __syncwarp();
            return true;
          }
          uint32_t ok = 1;
          if (elected) {
            steps(0, kEarlyKeys / 16);
            // the rest of P is usually written while the first steps run: the issuing lane
            // alone waits for it, so that the remaining steps follow on a still busy pipe
            ok = mbar_wait(&p_full[s], (sc - 1) & 1, tmo, abort_flag) ? 1u : 0u;
            if (ok) {
              tc_fence_after();
              steps(kEarlyKeys / 16, kBlockN / 16);
              if (last) publish();
              mma_commit(&v_empty[vs]);
            }
          }
          if (__shfl_sync(0xffffffffu, ok, 0) == 0) {
            fail();
            return false;
          }
          return true;
        };
        if constexpr (kSepP<D, kMode, kBias>) {
          // P in its own columns: S(x) follows the softmax's read of S(prev) (turn order on the
          // S groups), and PV(prev) follows P(prev), outside the turn order
          const uint32_t p_tmem = tmem + 384 + s * 64;
          int ja = 0, jb = 0, jm = 0;
          uint32_t k_grp = 0;
          bool s_pend = false, p_pend = false, first_pv = true;
          uint32_t prev = 0, prev_si = 0;  // ring position and S index of this tile's last S
          auto pv_sep = [&](uint32_t x, uint32_t si) -> bool {
            const int vs = x % C::kVStages;
            if (!wait_all(&v_full[vs], (x / C::kVStages) & 1)) return false;
            if (first_pv && !wait_all(&o_free[s], (oc & 1) ^ 1)) return false;
            if (!wait_all(&p_full[s], si & 1)) return false;
            tc_fence_after();
            if (elected) {
              const uint32_t vtile = v_base + vs * C::kTileBytes;
#pragma unroll
              for (int kk = 0; kk < kBlockN / 16; ++kk) {
                const uint64_t bdesc = smem_desc_sw128(vtile + kk * 16 * 128, kRegionBytes, 1024);
                mma_ts(o_tmem, p_tmem + kk * 8, bdesc, idesc_pv, (first_pv && kk == 0) ? 0u : 1u);
              }
              mma_commit(&v_empty[vs]);
              mma_commit(&p_free[s]);
            }
            __syncwarp();
            first_pv = false;
            return true;
          };
          for (;;) {
            const int na = w.t[0].next(ja), nb = w.t[1].next(jb);
            const int kb = min(na, nb);
            if (kb == kNone) break;
            const bool mine_tile = (s == 0 ? na : nb) == kb;
            const uint32_t x = g;
            const int ks = x % C::kKStages, vs = x % C::kVStages;
            if (!mine_tile) {
              // a key tile only the other query tile visits: the PV this tile owes, then release
              // the slots once they hold this key tile
              if (p_pend) {
                if (!pv_sep(prev, prev_si)) return;
                p_pend = false;
              }
              if (!wait_all(&k_full[ks], (x / C::kKStages) & 1)) return;
              if (elected) mbar_arrive(&k_empty[ks]);
              if (!wait_all(&v_full[vs], (x / C::kVStages) & 1)) return;
              if (elected) mbar_arrive(&v_empty[vs]);
            } else {
              if (!wait_all(&k_full[ks], (x / C::kKStages) & 1)) return;
              // S(x) overwrites S(prev): the softmax has read it
              if (s_pend && !wait_all(&p_early[s], prev_si & 1)) return;
              if (!turn_wait(before(k_grp))) return;
              tc_fence_after();
              if (elected) {
                const uint32_t ktile = k_base + ks * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                  const uint32_t off = (kk / 4) * kRegionBytes + (kk % 4) * 32;
                  mma_ss(s_tmem, smem_desc_sw128(qtile + off, 16, 1024), smem_desc_sw128(ktile + off, 16, 1024),
                         idesc_qk, kk > 0 ? 1u : 0u);
                }
                publish();
                mma_commit(&s_full[s]);
                mma_commit(&k_empty[ks]);
                if (jm + 1 == my_n) mma_commit(&q_empty[qslot]);
              }
              __syncwarp();
              ++mine;
              ++k_grp;
              const uint32_t si = sc++;
              ++jm;
              if (p_pend && !pv_sep(prev, prev_si)) return;
              s_pend = p_pend = true;
              prev = x;
              prev_si = si;
            }
            if (na == kb) ++ja;
            if (nb == kb) ++jb;
            ++g;
          }
          if (p_pend && !pv_sep(prev, prev_si)) return;
          // the next unit's first S overwrites this unit's last one once the softmax has read it
          if (s_pend && !wait_all(&p_early[s], prev_si & 1)) return;
          if (my_n > 0) {
            if (elected) mma_commit(&o_ready[s]);
            __syncwarp();
            ++oc;
          }
          base_o += groups_o;
          continue;
        }
        int ja = 0, jb = 0, jm = 0;
        uint32_t k_grp = 0;  // groups of this tile issued in this unit
        bool pend = false, first_pv = true;
        uint32_t prev = 0;
        for (;;) {
          const int na = w.t[0].next(ja), nb = w.t[1].next(jb);
          const int kb = min(na, nb);
          if (kb == kNone) break;
          const bool mine_tile = (s == 0 ? na : nb) == kb;
          const uint32_t x = g;
          const int ks = x % C::kKStages, vs = x % C::kVStages;
          if (!mine_tile) {
            // a key tile only the other query tile visits: first the PV this tile owes (its
            // V slot may be needed before this warp reaches its next own key tile), then
            // release the slots once they hold this key tile
            if (kMode != kModeStats && pend) {
              if (!pv_ready(prev, first_pv)) return;
              if (!turn_wait(before(k_grp))) return;
              if (!pv(prev, first_pv, true)) return;
              ++mine;
              ++k_grp;
              first_pv = false;
              pend = false;
            }
            if (!wait_all(&k_full[ks], (x / C::kKStages) & 1)) return;
            if (elected) mbar_arrive(&k_empty[ks]);
            if constexpr (kMode != kModeStats) {
              if (!wait_all(&v_full[vs], (x / C::kVStages) & 1)) return;
              if (elected) mbar_arrive(&v_empty[vs]);
            }
          } else {
            if (!wait_all(&k_full[ks], (x / C::kKStages) & 1)) return;
            if constexpr (kMode == kModeStats) {
              // S(x) overwrites S(prev): the softmax has read it (it arrives on p_full then)
              if (pend && !wait_all(&p_full[s], (sc - 1) & 1)) return;
            } else {
              if (pend && !pv_ready(prev, first_pv)) return;
            }
            if (!turn_wait(before(k_grp))) return;
            // PV of this tile's previous key tile first: S(x) overwrites the P it reads
            if (kMode != kModeStats && pend && !pv(prev, first_pv, false)) return;
            if (pend) first_pv = false;
            tc_fence_after();
            if (elected) {
              const uint32_t ktile = k_base + ks * C::kTileBytes;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                // A = Q, B = K: both K-major, 128-byte rows, 8-row groups 1024 bytes apart.
                const uint32_t off = (kk / 4) * kRegionBytes + (kk % 4) * 32;
                mma_ss(s_tmem, smem_desc_sw128(qtile + off, 16, 1024), smem_desc_sw128(ktile + off, 16, 1024),
                       idesc_qk, kk > 0 ? 1u : 0u);
              }
              publish();
              mma_commit(&s_full[s]);
              mma_commit(&k_empty[ks]);
              // the tile's last S: Q may be reloaded once it completes
              if (jm + 1 == my_n) mma_commit(&q_empty[qslot]);
            }
            __syncwarp();
            ++mine;
            ++k_grp;
            ++sc;
            ++jm;
            pend = true;
            prev = x;
          }
          if (na == kb) ++ja;
          if (nb == kb) ++jb;
          ++g;
        }
        if constexpr (kMode == kModeStats) {
          // the next unit's first S overwrites this unit's last one once the softmax has read it
          if (pend && !wait_all(&p_full[s], (sc - 1) & 1)) return;
        } else {
          if (pend) {
            if (!pv_ready(prev, first_pv)) return;
            if (!turn_wait(before(k_grp))) return;
            if (!pv(prev, first_pv, true)) return;
            ++mine;
            ++k_grp;
          }
          if (my_n > 0) {
            if (elected) mma_commit(&o_ready[s]);
            __syncwarp();
            ++oc;
          }
        }
        base_o += groups_o;
      }
    }();
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax + epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kSoftmaxRegs));
    [&] {
      const int s = warp / 4;            // stream (tile A or B)
      const int r = threadIdx.x % 128;   // query row within the tile = TMEM lane
      const uint32_t lane_addr = tmem + ((uint32_t)((warp % 4) * 32) << 16);
      const uint32_t scol = s * 128, ocol = 256 + s * D;
      const float sl2 = P.scale_log2;
      uint32_t sc = 0, oc = 0, bcs = 0;  // S tiles, units, bias tiles seen
      // Statistics pass with the weights fill: while query tile t of a (batch, head) is
      // processed, the stream's leader stores the zero tile over the key tiles past the bound of
      // the mirror tile nqt - 1 - t of the same (batch, head), 64 keys per TMA store (the tensor
      // map leaves out keys and rows past the array), a share after each key tile so that the
      // stores do not hold up the K loads in the TMA unit. Every tile is visited once, so every
      // tile's zeros are written once; mirrored, the largest fills (short causal rows) ride with
      // the longest rows, which run first, instead of piling up at the end of the launch.
      int fz_next = 0, fz_end = 0, fz_per = 0, fz_i0 = 0, fz_h = 0, fz_b = 0;
      auto fill_begin = [&](const Unit& uw, const QTile& uqt) {
        if (threadIdx.x % 128 != 0) return;
        BatchInfo bi;
        bi.q_len = uw.q_len;
        bi.kv_len = uw.kv_len;
        bi.offset = uw.offset;
        bi.skip = false;
        bi.q_rows = uw.q_rows;
        bi.q0 = bi.k0 = 0;
        const int nqt = (P.Lq + kBlockM - 1) / kBlockM;
        const QTile mq = make_qtile(P, bi, uqt.h, nqt - 1 - uqt.qt, true);
        fz_next = 2 * mq.n;
        fz_end = max((P.Lk + 63) / 64, fz_next);
        fz_per = uqt.n > 0 ? (fz_end - fz_next + uqt.n - 1) / uqt.n : fz_end - fz_next;
        fz_i0 = mq.i0;
        fz_h = mq.h;
        fz_b = uw.b;
      };
      auto fill_some = [&](int count) {
        if (threadIdx.x % 128 != 0 || fz_next >= fz_end) return;
        for (int x = 0; x < count && fz_next < fz_end; ++x, ++fz_next)
          tma_store_4d(&maps.w, v_smem, 64 * fz_next, fz_i0, fz_h, fz_b);
        bulk_commit();
      };
      uint32_t qi = 0;                   // Q tiles of both streams so far (ring position)
      for (uint32_t kq = 0;; ++kq) {
        int u;
        Unit w;
        if (!next_unit(kq, u, w)) return;
        if (u >= n_units) break;
        const QTile qt = s ? w.t[1] : w.t[0];
        const uint32_t my_qi = qi + ((s == 1 && w.t[0].n > 0) ? 1u : 0u);
        qi += (w.t[0].n > 0 ? 1u : 0u) + (w.t[1].n > 0 ? 1u : 0u);
        if (kMode == kModeAux && P.q_rope && qt.n > 0) {
          // Rotary embedding of this thread's query row in the tile's Q slot, once the tile
          // has landed: the pair (c, c + D/2) by the angle whose (cos, sin) the table holds
          // as fp16 for row b * Lq + i. 128-byte swizzle: logical 16-byte chunk x of row r
          // is stored at chunk x ^ (r % 8). The writes are made visible to the tensor core
          // (async proxy) before the warp releases the tile to its MMA warp.
          const int qslot = (int)(my_qi % C::kQSlots);
          if (!wait_all(&q_full[qslot], (my_qi / C::kQSlots) & 1)) return;
          if (qt.i0 + r < P.Lq)
            rotate_q_row<T, D>(q_smem + qslot * C::kTileBytes, r,
                               P.q_rope + ((long long)w.b * P.Lq + qt.i0 + r) * (D / 2));
          asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
          __syncwarp();
          if (lane == 0) mbar_arrive(&q_rot[qslot]);
        }
        if (qt.i0 == kNone) continue;  // the unit has no tile B
        const int i = qt.i0 + r;
        T* orow = out + ((w.o0 + i) * P.H + qt.h) * D;
        // range-checked build: a row this thread would store must lie inside out
        const bool row_ok = SDPA_CHECKED(P.status, i >= w.q_rows || (qt.h < P.H && w.o0 + i <
                                         (P.q_start ? (long long)P.Lq_total : (long long)P.B * P.Lq)));
        if (qt.n == 0) {
          // no key tile: NaN rows (nothing attended) or zero rows (past q_lengths)
          if constexpr (kMode == kModeAux || kMode == kModeStats) {
            if (P.lse && i < P.Lq) P.lse[((long long)w.b * P.H + qt.h) * P.Lq + i] = INFINITY;
          }
          if constexpr (kMode == kModeStats) {
            if (P.stats_fill && qt.i0 < P.Lq) {
              fill_begin(w, qt);
              fill_some(fz_per);
            }
            continue;  // the output is the weights pass's
          }
          if (i < w.q_rows && row_ok) {
            const float val = (i >= w.q_len) ? 0.f : __int_as_float(0x7fc00000);
            const uint32_t wv = std::is_same<T, __half>::value ? pack_f16x2(val, val) : pack_bf16x2(val, val);
#pragma unroll
            for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(wv, wv, wv, wv);
          }
          continue;
        }
        // keys j < row_lim are allowed by kv_lengths and the causal bound of this row; rows past
        // q_lengths (or the array) attend nothing, so no bias / mask element is read for them
        long long lim = (i < w.q_len) ? w.kv_len : 0;
        if (P.causal != SDPA_CAUSAL_NONE) lim = min(lim, (long long)w.offset + i + 1);
        const int row_lim = (int)max(lim, -1LL);
        const BT* bias_row = nullptr;
        if constexpr (kBias != kBiasNone)
          bias_row = static_cast<const BT*>(P.bias) + (long long)i * P.bs[1] + (long long)qt.h * P.bs[2] +
                     (long long)w.b * P.bs[3];
        const uint8_t* mask_row = nullptr;
        if constexpr (kMask == kMaskDense)
          mask_row = P.mask + (long long)i * P.ms[1] + (long long)qt.h * P.ms[2] + (long long)w.b * P.ms[3];
        float m_used = -INFINITY, l = 0.f;
        // weights pass: the row's log-sum-exp from the statistics pass (+inf: no key, or
        // padding) and the row's first position in the weights (the dropout counter)
        float row_lse = INFINITY;
        unsigned long long wbase = 0;
        if constexpr (kMode == kModeWeights) {
          const long long wr = ((long long)w.b * P.H + qt.h) * P.Lq + i;
          if (i < P.Lq) {
            row_lse = P.lse[wr];
            wbase = (unsigned long long)wr * (unsigned long long)P.Lk;
          }
          if (i < w.q_len && row_lse != INFINITY) l = 1.f;  // O is already normalised
        }
        if constexpr (kMode == kModeStats) {
          if (P.stats_fill) fill_begin(w, qt);
        }
        for (int j = 0; j < qt.n; ++j) {
          const int kb = qt.kb(j);
          const int key0 = kb * kBlockN;
          const int nvalid = min(max(row_lim - key0, 0), kBlockN);
          uint32_t bw[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
          if constexpr (kMask == kMaskBits) {
            if ((qt.list[j] >> 30) == SDPA_BLOCK_PARTIAL && nvalid > 0) {
              const int hm = P.bi_nheads == 1 ? 0 : qt.h;
              const long long blk = ((long long)hm * P.bi_nqb + qt.qt) * P.bi_nkb + kb;
              // range-checked build: the block must lie inside the classification
              if (SDPA_CHECKED(P.status, kb < P.bi_nkb && blk < (long long)P.bi_nheads * P.bi_nqb * P.bi_nkb)) {
                const uint4 b4 = *reinterpret_cast<const uint4*>(P.bbits + (blk * kBlockM + r) * 4);
                bw[0] = b4.x; bw[1] = b4.y; bw[2] = b4.z; bw[3] = b4.w;
              }
            }
          }
          if (!wait_all(&s_full[s], sc & 1)) return;
          ++sc;
          tc_fence_after();
          uint32_t v[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(lane_addr + scol + c * 32, v[c]);
          tmem_wait_ld();
          if constexpr (kMode == kModeStats) {
            // S is in registers: its columns are free for the next S
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[s]);
            if (P.stats_fill) fill_some(fz_per);
          }
          if constexpr (kSepP<D, kMode, kBias>) {
            // S is in registers: its columns are free for the next S
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_early[s]);
          }
          if constexpr (kMode == kModeWeights) {
            // w = 2^(s * scale*log2e - lse) on the attended keys, 0 elsewhere, NaN for a row
            // with no key. Dropout: the weight takes 16-bit field u of its group's draw; with f
            // the float 2^23 + u (u under the exponent bits of 2^23), sat(f + 1 - thr - 2^23) is
            // exactly 1 when u >= thr (kept) and 0 otherwise, and the kept weight's 1/(1 - p) is
            // in the exponent. Keys past the row's bound are zeroed after the 16-bit packing,
            // on the tiles where a row of the warp has such keys. w' goes into TMEM for the PV
            // MMA; the weights go through the warp's part of the staging tile to TMA stores.
            const bool nan_row = i < w.q_len && row_lse == INFINITY;
            const bool drop = P.drop_thr > 0;
            const float negl = nan_row ? 0.f : -row_lse + (drop ? log2f(P.inv_keep) : 0.f);
            const float kthr = 1.f - (float)P.drop_thr - 8388608.f;
            // One 64-key half of the warp's 32 rows (v[hh]: this thread's row) in the 128-byte
            // swizzle (16-byte chunk x of row r at x ^ (r % 8)), once the warp's previous store
            // has read its 4 KB; lane 0 then stores it with TMA, which leaves out rows and keys
            // past the array. Both halves go out after P is handed over, while the MMAs run.
            uint8_t* stg = o_stage + s * (C::kOStageBytes / 2) + (warp % 4) * (32 * 128);
            const int wrow0 = qt.i0 + 32 * (warp % 4);
            auto stage_half = [&](int hh) {
              if (lane == 0) bulk_wait_read();
              __syncwarp();
              const uint32_t nanw = std::is_same<T, __half>::value ? 0x7E007E00u : 0x7FC07FC0u;
#pragma unroll
              for (int x = 0; x < 8; ++x) {
                const uint4 st = nan_row ? make_uint4(nanw, nanw, nanw, nanw)
                                         : make_uint4(v[hh][4 * x], v[hh][4 * x + 1], v[hh][4 * x + 2], v[hh][4 * x + 3]);
                *reinterpret_cast<uint4*>(stg + lane * 128 + ((x ^ (lane & 7)) << 4)) = st;
              }
              asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
              __syncwarp();
              // range-checked build: a half outside the weights is reported and not stored
              if (lane == 0 && key0 + 64 * hh < P.Lk && wrow0 < P.Lq &&
                  SDPA_CHECKED(P.status, qt.h < P.H && w.b < P.B)) {
                tma_store_4d(&maps.w_warp, stg, key0 + 64 * hh, wrow0, qt.h, w.b);
                bulk_commit();
              }
            };
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int lim = nvalid - 32 * c;
              // the 8 groups of these 32 keys: consecutive draws, one gamma apart in the state
              unsigned long long z = drop ? dropout_state(P.drop_seed, (wbase + (unsigned long long)(key0 + 32 * c)) >> 2) : 0ull;
              uint32_t pk[16];
#pragma unroll
              for (int gq = 0; gq < 8; ++gq) {
                float mk[4] = {1.f, 1.f, 1.f, 1.f};
                if (drop) {
                  const unsigned long long rr = splitmix64_mix(z);
                  z += kSplitMixGamma;
                  const uint32_t lo = (uint32_t)rr, hi = (uint32_t)(rr >> 32);
                  mk[0] = __saturatef(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7610)) + kthr);
                  mk[1] = __saturatef(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7632)) + kthr);
                  mk[2] = __saturatef(__uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7610)) + kthr);
                  mk[3] = __saturatef(__uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7632)) + kthr);
                }
                const int e = 4 * gq;
                float x0, x1, x2, x3;
                fma2(x0, x1, __uint_as_float(v[c][e]), __uint_as_float(v[c][e + 1]), sl2, sl2, negl, negl);
                fma2(x2, x3, __uint_as_float(v[c][e + 2]), __uint_as_float(v[c][e + 3]), sl2, sl2, negl, negl);
                const float p0 = ex2(x0) * mk[0], p1 = ex2(x1) * mk[1], p2 = ex2(x2) * mk[2], p3 = ex2(x3) * mk[3];
                pk[2 * gq] = std::is_same<T, __half>::value ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1);
                pk[2 * gq + 1] = std::is_same<T, __half>::value ? pack_f16x2(p2, p3) : pack_bf16x2(p2, p3);
              }
              if (__any_sync(0xffffffffu, lim < 32)) {
                // keys [lim, 32) of this chunk are past the row's bound (their exponentials
                // may be anything): the pair (2e, 2e + 1) keeps what lies below lim
#pragma unroll
                for (int e = 0; e < 16; ++e)
                  pk[e] = 2 * e + 1 < lim ? pk[e] : (2 * e < lim ? (pk[e] & 0xFFFFu) : 0u);
              }
#pragma unroll
              for (int e = 0; e < 16; ++e) v[c / 2][(c % 2) * 16 + e] = pk[e];
            }
            tmem_st32(lane_addr + scol, v[0]);
            tmem_st32(lane_addr + scol + 32, v[1]);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if constexpr (kSplitP<D, kMode, kBias>) mbar_arrive(&p_early[s]);
              mbar_arrive(&p_full[s]);
            }
            stage_half(0);
            stage_half(1);
            continue;
          }
          // Fast path (no bias, no mask bytes, every key of the tile attended by every row of
          // the warp): v keeps the raw scores, the max is taken on them (scale > 0) and the
          // exponent argument is one packed FMA, s * scale*log2e - m. Otherwise v becomes the
          // logits in log2 units, -inf where masked, and the argument is v - m.
          float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          const bool full_row = (nvalid == kBlockN) && (kMask == kMaskNone ||
                                (kMask == kMaskBits && (bw[0] & bw[1] & bw[2] & bw[3]) == 0xffffffffu));
          const bool fast = kBias == kBiasNone && kMask != kMaskDense && __all_sync(0xffffffffu, full_row);
          float mul;
          const int bslot = s * C::kBiasSlots + (int)(bcs % C::kBiasSlots);
          const uint8_t* bsm = b_smem + bslot * C::kBiasTileBytes;
          if constexpr (kBias == kBiasTile) {
            if (!wait_all(&b_full[bslot], (bcs / C::kBiasSlots) & 1)) return;
          }
          if (kBias == kBiasNone && kMask != kMaskDense) {
            // No bias: the raw scores stay raw (the max commutes with scale > 0) and a masked
            // key only has to become -inf; one keep-word per 32 keys drives the selects.
            mul = sl2;
            if (!fast) {
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const int lim = nvalid - 32 * c;
                uint32_t keep = lim >= 32 ? 0xffffffffu : (lim <= 0 ? 0u : (1u << lim) - 1u);
                if constexpr (kMask == kMaskBits) keep &= bw[c];
#pragma unroll
                for (int e = 0; e < 32; ++e) v[c][e] = ((keep >> e) & 1u) ? v[c][e] : 0xff800000u;
              }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int e = 0; e < 32; e += 2)
                mx[(e >> 1) & 3] = fmax3(mx[(e >> 1) & 3], __uint_as_float(v[c][e]), __uint_as_float(v[c][e + 1]));
          } else if constexpr (kBias != kBiasNone && kMask != kMaskDense) {
            // With a bias: the logits stay in natural units, x = s * scale + b (one packed FMA
            // per pair), and the factor log2(e) goes into the exponent's FMA (mul). A masked key
            // (past the row's bound, or a zero bit of a partial block) becomes -inf, in the
            // chunks where some row of the warp has one.
            mul = kLog2e;
            const float scl = P.scale;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int lim = nvalid - 32 * c;
              uint32_t keep = lim >= 32 ? 0xffffffffu : (lim <= 0 ? 0u : (1u << lim) - 1u);
              if constexpr (kMask == kMaskBits) keep &= bw[c];
              float bias32[32];
#pragma unroll
              for (int e = 0; e < 32; e += 8) {
                const int col = c * 32 + e;
                float* f8 = bias32 + e;
                if constexpr (kBias == kBiasTile) {
                  // 128-byte swizzled rows: 16-byte chunk ch of row r sits at chunk ch ^ (r % 8)
                  const int box = col >> 6, ch = (col & 63) >> 3;
                  load8<BT>(reinterpret_cast<const BT*>(bsm + box * kRegionBytes + r * 128 + ((ch ^ (r & 7)) << 4)),
                            *reinterpret_cast<float(*)[8]>(f8));
                } else if (col + 8 <= nvalid) {
                  load8<BT>(bias_row + key0 + col, *reinterpret_cast<float(*)[8]>(f8));
                } else {
#pragma unroll
                  for (int k = 0; k < 8; ++k) f8[k] = (col + k < nvalid) ? to_f32(bias_row[key0 + col + k]) : 0.f;
                }
              }
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                float t0, t1;
                fma2(t0, t1, __uint_as_float(v[c][e]), __uint_as_float(v[c][e + 1]), scl, scl, bias32[e], bias32[e + 1]);
                v[c][e] = __float_as_uint(t0);
                v[c][e + 1] = __float_as_uint(t1);
              }
              if (__any_sync(0xffffffffu, keep != 0xffffffffu)) {
#pragma unroll
                for (int e = 0; e < 32; ++e) v[c][e] = ((keep >> e) & 1u) ? v[c][e] : 0xff800000u;
              }
#pragma unroll
              for (int e = 0; e < 32; e += 2)
                mx[(e >> 1) & 3] = fmax3(mx[(e >> 1) & 3], __uint_as_float(v[c][e]), __uint_as_float(v[c][e + 1]));
            }
          } else {
            mul = 1.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float bia[32];
              uint32_t mk[8];
              if constexpr (kBias != kBiasNone) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                  const int col = c * 32 + e;
                  float f8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                  if constexpr (kBias == kBiasTile) {
                    // 128-byte swizzled rows: 16-byte chunk ch of row r sits at chunk ch ^ (r % 8)
                    const int box = col >> 6, ch = (col & 63) >> 3;
                    load8<BT>(reinterpret_cast<const BT*>(bsm + box * kRegionBytes + r * 128 + ((ch ^ (r & 7)) << 4)), f8);
                  } else if (col + 8 <= nvalid) {
                    load8<BT>(bias_row + key0 + col, f8);
                  } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                      if (col + k < nvalid) f8[k] = to_f32(bias_row[key0 + col + k]);
                  }
#pragma unroll
                  for (int k = 0; k < 8; ++k) bia[e + k] = f8[k] * kLog2e;
                }
              }
              if constexpr (kMask == kMaskDense) {
                const int col = c * 32;
                if (col + 32 <= nvalid) {
                  const uint4 a = *reinterpret_cast<const uint4*>(mask_row + key0 + col);
                  const uint4 b = *reinterpret_cast<const uint4*>(mask_row + key0 + col + 16);
                  mk[0] = a.x; mk[1] = a.y; mk[2] = a.z; mk[3] = a.w; mk[4] = b.x; mk[5] = b.y; mk[6] = b.z; mk[7] = b.w;
                } else {
#pragma unroll
                  for (int k = 0; k < 8; ++k) {
                    uint32_t wd = 0;
#pragma unroll
                    for (int y = 0; y < 4; ++y)
                      if (col + 4 * k + y < nvalid) wd |= (uint32_t)(mask_row[key0 + col + 4 * k + y] != 0) << (8 * y);
                    mk[k] = wd;
                  }
                }
              }
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const int col = c * 32 + e;
                float t = __uint_as_float(v[c][e]) * sl2;
                if constexpr (kBias != kBiasNone) t += bia[e];
                bool ok = col < nvalid;
                if constexpr (kMask == kMaskBits) ok = ok && ((bw[c] >> e) & 1u);
                if constexpr (kMask == kMaskDense) ok = ok && ((mk[e / 4] >> (8 * (e % 4))) & 0xFFu);
                t = ok ? t : -INFINITY;
                v[c][e] = __float_as_uint(t);
                mx[e & 3] = fmaxf(mx[e & 3], t);
              }
            }
          }
          if constexpr (kBias == kBiasTile) {
            __syncwarp();  // every lane of the warp has read its bias row
            if (lane == 0) mbar_arrive(&b_empty[bslot]);
            ++bcs;
          }
          const float rmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * mul;
          // the running max moves only when the row max passes it by 2^8 (or leaves -inf)
          const bool grow = (rmax > m_used + kRescaleThreshold) || (m_used == -INFINITY && rmax != -INFINITY);
          // O needs rescaling when it holds terms taken against a finite max (alpha may
          // underflow to 0 when the max jumps by more than 2^126: O is then cleared)
          const bool had_max = m_used != -INFINITY;
          float alpha = 1.f;
          if (grow) {
            alpha = had_max ? ex2(m_used - rmax) : 0.f;
            m_used = rmax;
          }
          const bool need_o = grow && had_max && j > 0;
          // O holds PV of the earlier key tiles (complete: the S commit covered them; with P in
          // its own columns the last PV is waited for here)
          if constexpr (kMode != kModeStats) {
            if (__any_sync(0xffffffffu, need_o)) {
              if constexpr (kSepP<D, kMode, kBias>) {
                if (!wait_all(&p_free[s], (sc - 2) & 1)) return;
                tc_fence_after();
              }
              rescale_o<D>(lane_addr + ocol, need_o ? alpha : 1.f);
            }
          }
          l *= alpha;
          const float negm = (m_used == -INFINITY) ? 0.f : -m_used;
          // P = 2^(v * mul - m), 16-bit pairs into the first 64 columns of the tile's S columns.
          float rs[4] = {0.f, 0.f, 0.f, 0.f};
          if constexpr (kMode == kModeStats) {
            // the row sum alone
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                float x0, x1;
                fma2(x0, x1, __uint_as_float(v[c][e]), __uint_as_float(v[c][e + 1]), mul, mul, negm, negm);
                add2(rs[(e >> 1) & 2], rs[((e >> 1) & 2) + 1], rs[(e >> 1) & 2], rs[((e >> 1) & 2) + 1], ex2(x0), ex2(x1));
              }
            l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
            continue;
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float x0, x1;
              fma2(x0, x1, __uint_as_float(v[c][e]), __uint_as_float(v[c][e + 1]), mul, mul, negm, negm);
              const float p0 = ex2(x0), p1 = ex2(x1);
              add2(rs[(e >> 1) & 2], rs[((e >> 1) & 2) + 1], rs[(e >> 1) & 2], rs[((e >> 1) & 2) + 1], p0, p1);
              pk[e / 2] = std::is_same<T, __half>::value ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1);
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) v[c / 2][(c % 2) * 16 + e] = pk[e];
            if (kSplitP<D, kMode, kBias> && c == kEarlyKeys / 32 - 1) {
              // keys [0, kEarlyKeys): 16-bit pairs in columns [0, kEarlyKeys / 2)
              static_assert(kEarlyKeys == 96, "P columns stored early: 32 + 16");
              tmem_st32(lane_addr + scol, v[0]);
              tmem_st16(lane_addr + scol + 32, *reinterpret_cast<const uint32_t(*)[16]>(&v[1][0]));
              tmem_wait_st();
              tc_fence_before();
              __syncwarp();  // the warp's stores are done (each lane waited for its own)
              if (lane == 0) mbar_arrive(&p_early[s]);
            }
          }
          l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
          if constexpr (kSepP<D, kMode, kBias>) {
            // P's columns are free once the PV of this stream's last P has completed (the
            // unit's first P follows the previous unit's output, which waited for all of them)
            if (j > 0) {
              if (!wait_all(&p_free[s], (sc - 2) & 1)) return;
              tc_fence_after();
            }
            const uint32_t pcol = 384 + s * 64;
            tmem_st32(lane_addr + pcol, v[0]);
            tmem_st32(lane_addr + pcol + 32, v[1]);
          } else if constexpr (kSplitP<D, kMode, kBias>) {
            tmem_st16(lane_addr + scol + kEarlyKeys / 2, *reinterpret_cast<const uint32_t(*)[16]>(&v[1][16]));
          } else {
            tmem_st32(lane_addr + scol, v[0]);
            tmem_st32(lane_addr + scol + 32, v[1]);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[s]);
        }
        if constexpr (kMode == kModeStats) {
          // the row's log-sum-exp in log2 units times lse_out_mul (+inf: no key, or padding)
          if (i < P.Lq)
            P.lse[((long long)w.b * P.H + qt.h) * P.Lq + i] =
                (i < w.q_len && l > 0.f) ? (m_used + log2f(l)) * P.lse_out_mul : INFINITY;
          if (P.stats_fill) fill_some(fz_end);
          continue;
        }
        if (!wait_all(&o_ready[s], oc & 1)) return;
        ++oc;
        tc_fence_after();
        const bool pad = i >= w.q_len;
        const float inv = (l > 0.f) ? 1.f / l : __int_as_float(0x7fc00000);
        if constexpr (kMode == kModeAux) {
          // the row's log-sum-exp in log2 units, for a weights pass that follows
          if (P.lse && i < P.Lq)
            P.lse[((long long)w.b * P.H + qt.h) * P.Lq + i] =
                (!pad && l > 0.f) ? (m_used + log2f(l)) * P.lse_out_mul : INFINITY;
        }
        bool staged = false;
        if constexpr (kOStage<D, kMode>) staged = P.q_start == nullptr;
        if (staged) {
          // Per 64-dim half: once the stream's staging tile is free (the leader thread's last
          // store has read it), each thread writes its row, scaled and rounded, in the 128-byte
          // swizzle (16-byte chunk x of row r at x ^ (r % 8)); the leader then stores the tile
          // with TMA, which leaves out rows past the tensor unwritten.
          uint8_t* stg = o_stage + s * (C::kOStageBytes / 2);
          const bool leader = (threadIdx.x % 128) == 0;
#pragma unroll 1
          for (int hh = 0; hh < D / 64; ++hh) {
            if (leader) {
              bulk_wait_read();
              mbar_arrive(&stage_free[s]);
            }
            // (two halves per unit, in every unit of the launch: the phase of half hh is hh % 2)
            if (!wait_all(&stage_free[s], hh & 1)) return;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              uint32_t o[32];
              tmem_ld32(lane_addr + ocol + hh * 64 + cc * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int xx = 0; xx < 4; ++xx) {
                const int x = 4 * cc + xx;  // 16-byte chunk of the row's 64 dims
                uint32_t wv[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const float a0 = pad ? 0.f : (l > 0.f ? __uint_as_float(o[8 * xx + 2 * k]) * inv : inv);
                  const float a1 = pad ? 0.f : (l > 0.f ? __uint_as_float(o[8 * xx + 2 * k + 1]) * inv : inv);
                  wv[k] = std::is_same<T, __half>::value ? pack_f16x2(a0, a1) : pack_bf16x2(a0, a1);
                }
                *reinterpret_cast<uint4*>(stg + r * 128 + ((x ^ (r & 7)) << 4)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
              }
            }
            asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&stage_full[s]);
            if (warp % 4 == 0) {
              if (!wait_all(&stage_full[s], hh & 1)) return;
              if (leader) {
                int oh = qt.h, orow0 = w.tq + qt.i0, ob = w.tb;
                // range-checked build: a tile outside out is reported and not stored
                if (SDPA_CHECKED(P.status, oh < P.H && orow0 < P.Lq && ob < P.B)) {
                  tma_store_4d(&maps.o, stg, hh * 64, oh, orow0, ob);
                  bulk_commit();
                }
              }
              __syncwarp();
            }
          }
        } else
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_addr + ocol + c * 32, o);
          tmem_wait_ld();
          if (i < w.q_rows && row_ok) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint32_t wv[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float a0 = pad ? 0.f : (l > 0.f ? __uint_as_float(o[e + 2 * k]) * inv : inv);
                const float a1 = pad ? 0.f : (l > 0.f ? __uint_as_float(o[e + 2 * k + 1]) * inv : inv);
                wv[k] = std::is_same<T, __half>::value ? pack_f16x2(a0, a1) : pack_bf16x2(a0, a1);
              }
              *reinterpret_cast<uint4*>(orow + c * 32 + e) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_free[s]);
      }
    }();
    // the staged output stores complete (their shared-memory source lives until then), also
    // when the role ended on a timeout
    if constexpr (kStageSmem<D, kMode> || kMode == kModeStats) {
      if (threadIdx.x % 128 == 0 || (kMode == kModeWeights && lane == 0)) bulk_wait();
    }
  }
  if (warp == kMmaWarpA || warp == kMmaWarpB) {
    // every MMA this CTA issued has completed before its TMEM is released (also on a timeout)
    if (elected) mma_commit(drain);
    __syncwarp();
    mbar_wait(drain, 0, tmo, nullptr);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarpA) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  // the last CTA to finish resets the unit counter for the next launch on this workspace
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(sched + 1, 1u) == gridDim.x - 1) {
      atomicExch(sched, 0u);
      atomicExch(sched + 1, 0u);
      __threadfence();
    }
  }
}

// Host launcher for one (T, D) pair; defined in the per-type translation units. bias_tiles:
// maps.bias describes the bias and the kBiasTile variant may be used (head_dim 64 only).
template <typename T, int D>
cudaError_t launch(const TensorMaps& maps, const Problem& P, void* out, int grid, bool bias_tiles,
                   cudaStream_t stream);
template <> cudaError_t launch<__nv_bfloat16, 128>(const TensorMaps&, const Problem&, void*, int, bool, cudaStream_t);
template <> cudaError_t launch<__nv_bfloat16, 64>(const TensorMaps&, const Problem&, void*, int, bool, cudaStream_t);
template <> cudaError_t launch<__half, 128>(const TensorMaps&, const Problem&, void*, int, bool, cudaStream_t);
template <> cudaError_t launch<__half, 64>(const TensorMaps&, const Problem&, void*, int, bool, cudaStream_t);

// The weights pass (kModeWeights, no bias or mask) for one (T, D) pair, after the statistics pass
// has written P.lse and the weights of the key tiles the pass does not visit have been written
// (by the statistics pass or weights_fill_kernel).
template <typename T, int D>
cudaError_t launch_weights(const TensorMaps& maps, const Problem& P, void* out, int grid, cudaStream_t stream);
// The forward with the row log-sum-exp (P.lse) and / or the rotated Q tiles (P.q_rope); no bias
// or mask.
template <typename T, int D>
cudaError_t launch_aux(const TensorMaps& maps, const Problem& P, void* out, int grid, cudaStream_t stream);
template <> cudaError_t launch_aux<__nv_bfloat16, 128>(const TensorMaps&, const Problem&, void*, int, cudaStream_t);
template <> cudaError_t launch_aux<__nv_bfloat16, 64>(const TensorMaps&, const Problem&, void*, int, cudaStream_t);
template <> cudaError_t launch_aux<__half, 128>(const TensorMaps&, const Problem&, void*, int, cudaStream_t);
template <> cudaError_t launch_aux<__half, 64>(const TensorMaps&, const Problem&, void*, int, cudaStream_t);
template <> cudaError_t launch_weights<__nv_bfloat16, 128>(const TensorMaps&, const Problem&, void*, int, cudaStream_t);
template <> cudaError_t launch_weights<__nv_bfloat16, 64>(const TensorMaps&, const Problem&, void*, int, cudaStream_t);
template <> cudaError_t launch_weights<__half, 128>(const TensorMaps&, const Problem&, void*, int, cudaStream_t);
template <> cudaError_t launch_weights<__half, 64>(const TensorMaps&, const Problem&, void*, int, cudaStream_t);
// Each row's log-sum-exp alone (kModeStats) into P.lse, for the weights pass
template <typename T, int D>
cudaError_t launch_stats(const TensorMaps& maps, const Problem& P, void* out, int grid, cudaStream_t stream);
template <> cudaError_t launch_stats<__nv_bfloat16, 128>(const TensorMaps&, const Problem&, void*, int, cudaStream_t);
template <> cudaError_t launch_stats<__nv_bfloat16, 64>(const TensorMaps&, const Problem&, void*, int, cudaStream_t);
template <> cudaError_t launch_stats<__half, 128>(const TensorMaps&, const Problem&, void*, int, cudaStream_t);
template <> cudaError_t launch_stats<__half, 64>(const TensorMaps&, const Problem&, void*, int, cudaStream_t);

// The weights of the key tiles a query tile does not visit (past its causal / kv_lengths bound,
// the tiles make_qtile leaves out): 0, or NaN for a row with no key. Grid (query tiles, H, B);
// kv_len is a multiple of 8, so each row's run starts on a 16-byte boundary.
template <typename T>
__global__ void __launch_bounds__(256) weights_fill_kernel(const Problem P) {
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const BatchInfo bi = resolve_batch(P, b);
  const QTile x = make_qtile(P, bi, h, qt, true);
  const int col0 = x.n * kBlockN;
  if (col0 >= P.Lk) return;
  const int chunks = (P.Lk - col0) / 8;  // 16-byte runs per row
  const int rows = min(kBlockM, P.Lq - qt * kBlockM);
  const uint32_t nanw = std::is_same<T, __half>::value ? 0x7E007E00u : 0x7FC07FC0u;
  T* base = static_cast<T*>(P.weights);
  for (int idx = threadIdx.x; idx < rows * chunks; idx += blockDim.x) {
    const int r = idx / chunks, c = idx % chunks;
    const int i = qt * kBlockM + r;
    long long lim = (i < bi.q_len) ? bi.kv_len : 0;
    if (P.causal != SDPA_CAUSAL_NONE) lim = min(lim, (long long)bi.offset + i + 1);
    const bool nan_row = i < bi.q_len && lim <= 0;
    T* row = base + (((long long)b * P.H + h) * P.Lq + i) * P.Lk + col0;
    reinterpret_cast<uint4*>(row)[c] = nan_row ? make_uint4(nanw, nanw, nanw, nanw) : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <typename T, int D, int kBias, int kMask, int kMode = kModeForward>
cudaError_t launch_variant(const TensorMaps& maps, const Problem& P, void* out, int grid, cudaStream_t stream) {
  auto kern = prefill_kernel<T, D, kBias, kMask, kMode>;
  const int smem = Cfg<D, kBias == kBiasTile>::smem_bytes(kStageSmem<D, kMode>);
  // checked and configured once per device (bit d of `ready`)
  static std::atomic<unsigned long long> ready{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
  if (!(ready.load(std::memory_order_acquire) & bit)) {
    cudaFuncAttributes attr;
    e = cudaFuncGetAttributes(&attr, kern);
    if (e != cudaSuccess) return e;
    // setmaxnreg.inc would wait forever if the launch held fewer registers than the split needs
    if (attr.numRegs < kLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    ready.fetch_or(bit, std::memory_order_acq_rel);
  }
  const int n_units = units_per_level(P) * n_levels(P);
  kern<<<grid, kThreads, smem, stream>>>(maps, P, static_cast<T*>(out), n_units);
  return cudaGetLastError();
}

inline int bias_variant(const Problem& P, bool bias_tiles) {
  if (!P.bias) return kBiasNone;
  if (P.bias_dtype == SDPA_F32) return kBiasF32;
  return bias_tiles ? kBiasTile : kBiasSame;
}
inline int mask_variant(const Problem& P) {
  if (P.bcls) return kMaskBits;
  if (P.mask) return kMaskDense;
  return kMaskNone;
}

#define SDPA_PREFILL_DEFINE_LAUNCH(T, D)                                                              \
  template <>                                                                                       \
  cudaError_t launch_aux<T, D>(const TensorMaps& maps, const Problem& P, void* out, int grid,      \
                               cudaStream_t stream) {                                               \
    return launch_variant<T, D, kBiasNone, kMaskNone, kModeAux>(maps, P, out, grid, stream);       \
  }                                                                                                 \
  template <>                                                                                       \
  cudaError_t launch_weights<T, D>(const TensorMaps& maps, const Problem& P, void* out, int grid,  \
                                   cudaStream_t stream) {                                           \
    return launch_variant<T, D, kBiasNone, kMaskNone, kModeWeights>(maps, P, out, grid, stream);   \
  }                                                                                                 \
  template <>                                                                                       \
  cudaError_t launch_stats<T, D>(const TensorMaps& maps, const Problem& P, void* out, int grid,    \
                                 cudaStream_t stream) {                                             \
    return launch_variant<T, D, kBiasNone, kMaskNone, kModeStats>(maps, P, out, grid, stream);     \
  }                                                                                                 \
  template <>                                                                                       \
  cudaError_t launch<T, D>(const TensorMaps& maps, const Problem& P, void* out, int grid,         \
                           bool bias_tiles, cudaStream_t stream) {                                  \
    const int b = bias_variant(P, bias_tiles && D == 64), m = mask_variant(P);                      \
    if constexpr (D == 64) {                                                                        \
      if (b == kBiasTile) {                                                                         \
        if (m == kMaskNone) return launch_variant<T, D, kBiasTile, kMaskNone>(maps, P, out, grid, stream); \
        if (m == kMaskDense) return launch_variant<T, D, kBiasTile, kMaskDense>(maps, P, out, grid, stream); \
        return launch_variant<T, D, kBiasTile, kMaskBits>(maps, P, out, grid, stream);              \
      }                                                                                             \
    }                                                                                               \
    switch (b * 3 + m) {                                                                            \
      case 0: return launch_variant<T, D, kBiasNone, kMaskNone>(maps, P, out, grid, stream);        \
      case 1: return launch_variant<T, D, kBiasNone, kMaskDense>(maps, P, out, grid, stream);       \
      case 2: return launch_variant<T, D, kBiasNone, kMaskBits>(maps, P, out, grid, stream);        \
      case 3: return launch_variant<T, D, kBiasSame, kMaskNone>(maps, P, out, grid, stream);        \
      case 4: return launch_variant<T, D, kBiasSame, kMaskDense>(maps, P, out, grid, stream);       \
      case 5: return launch_variant<T, D, kBiasSame, kMaskBits>(maps, P, out, grid, stream);        \
      case 6: return launch_variant<T, D, kBiasF32, kMaskNone>(maps, P, out, grid, stream);         \
      case 7: return launch_variant<T, D, kBiasF32, kMaskDense>(maps, P, out, grid, stream);        \
      default: return launch_variant<T, D, kBiasF32, kMaskBits>(maps, P, out, grid, stream);       \
    }                                                                                               \
  }

}  // namespace prefill
}  // namespace sdpa
