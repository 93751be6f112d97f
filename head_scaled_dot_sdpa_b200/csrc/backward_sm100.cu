// The gradient of the fused implementation on the fifth-generation tensor cores (Flux.jl page
// "Neural Network primitives from NNlib.jl", entry scaled_dot_product_attention, paragraph
// "Fused implementation": a gradient with respect to query, key, value and scale that
// recomputes the weights tile by tile; a query whose output is NaN takes no part).
//
// For the loss sum(dout . out), with w_ij = 2^(s_ij scale log2e - lse_i) (s_ij = q_i . k_j, lse
// the row log-sum-exp in log2 units that the forward leaves), dp_ij = dout_i . v_j and
// delta_i = dout_i . out_i:
//     dx_ij = w_ij (dp_ij - delta_i),
//     dv_j = sum_i w_ij dout_i,  dk_j = scale sum_i dx_ij q_i,  dq_i = scale sum_j dx_ij k_j,
//     dscale = sum_ij dx_ij s_ij.
// bf16 / fp16 with head_dim = v_head_dim = 128, no bias, mask or block info; three kernels after
// the forward (which writes lse):
//  - bwd_delta_kernel: delta = dout . out per row;
//  - bwd_kv_kernel: one (key tile of 128, kv head, batch) per unit; for every query tile of
//    every query head of the group that sees the key tile: S^T = K Q^T and dP^T = V dout^T into
//    TMEM (tcgen05.mma, operands in shared memory by TMA), then w^T and dx^T by the elementwise
//    warps, written back over S^T / dP^T, then dV += w^T dout and dK += dx^T Q (tcgen05.mma with
//    the A operand in TMEM). dK and dV stay in TMEM over the whole unit: each row is written once.
//  - bwd_q_kernel: one (query tile of 128, head, batch) per unit; for every key tile it sees:
//    S = Q K^T and dP = dout V^T, dx by the elementwise warps (and dscale), dQ += dx K.
// dx is held as a bf16 / fp16 high part plus the rounded remainder (two MMAs), so the dK and
// dQ products keep about 16 significant bits: one 16-bit rounding of dx loses too much where
// the sum over a row cancels (sum_j dx_ij = 0). w >= 0 enters dV with one rounding (its sum
// does not cancel: a relative error near 2^-9 / sqrt(3)).
// TMEM columns (512): bwd_kv: S^T [0,128), dP^T [128,256), dV [256,384), dK [384,512);
// bwd_q: S [0,128) and [384,512) (alternate key tiles), dP [128,256), dQ [256,384). A 32-column chunk of S (or dP) receives, once
// read, the high parts of its 32 values (16 columns of 16-bit pairs) then the low parts (w^T:
// the high parts only).
// Warp roles (384 threads): warps 0-7 elementwise (warp w: TMEM lanes 32 (w % 4).., value
// columns 64 (w / 4)..), warp 8 TMA producer, warp 9 MMA issuer and TMEM owner. Every
// mbarrier wait is bounded; on a timeout the CTA records SDPA_ERR_TIMEOUT and unwinds.
#include <cuda.h>

#include <algorithm>
#include <atomic>
#include <type_traits>

#include "device_common.cuh"
#include "sm100_primitives.cuh"
#include "tma_map.h"

namespace sdpa {
namespace bwd {

using namespace sm100;

constexpr int kD = 128;                 // head_dim = v_head_dim
constexpr int kBlk = 128;               // rows of a query / key tile
constexpr int kThreads = 384;
constexpr int kEw = 8;                  // elementwise warps
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kRegion = 128 * 128;      // 128 rows x 64 16-bit columns (128-byte rows)
constexpr int kTile = 2 * kRegion;      // 128 rows x 128 columns
constexpr uint32_t kTmemCols = 512;
constexpr int kEwRegs = 216, kOtherRegs = 72, kLaunchRegs = 168;
static_assert(2 * 128 * kEwRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs, "register split");
// shared memory: 6 tiles, lse / delta staging (2 slots x 2 x 128 floats), barriers, TMEM slot
constexpr int kSmemBytes = 6 * kTile + 2 * 2 * kBlk * 4 + 32 * 8 + 64 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

struct Maps {
  CUtensorMap q, k, v, dout;
};

// key tiles [0, kt_end) a query tile sees; query tiles [qt_begin, qt_end) a key tile is seen by
__device__ __forceinline__ int kt_end_of(const Problem& P, const BatchInfo& bi, int qt) {
  if (bi.q_len <= qt * kBlk) return 0;
  long long lim = bi.kv_len;
  if (P.causal != SDPA_CAUSAL_NONE) {
    const long long last_row = min(qt * kBlk + kBlk - 1, bi.q_len - 1);
    lim = min(lim, (long long)bi.offset + last_row + 1);
  }
  return lim <= 0 ? 0 : (int)((lim + kBlk - 1) / kBlk);
}
__device__ __forceinline__ void qt_range_of(const Problem& P, const BatchInfo& bi, int kt, int& qb, int& qe) {
  qb = 0;
  qe = 0;
  if (kt * kBlk >= bi.kv_len || bi.q_len <= 0) return;
  qe = (bi.q_len + kBlk - 1) / kBlk;
  if (P.causal != SDPA_CAUSAL_NONE) {
    // the first row that sees key kt*128 is kt*128 - offset
    const long long first = (long long)kt * kBlk - bi.offset;
    qb = first <= 0 ? 0 : (int)min((long long)qe, first / kBlk);
  }
}

// Bounded waits shared by the roles (as in the forward kernel).
struct Waiter {
  volatile int* abort;
  int* status;
  uint64_t tmo;
  __device__ __forceinline__ void fail() const {
    *abort = 1;
    report(status, SDPA_ERR_TIMEOUT);
  }
  __device__ __forceinline__ bool all(uint64_t* bar, uint32_t parity) const {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    const bool ok = mbar_wait(bar, parity, tmo, abort);
    if (__all_sync(0xffffffffu, ok)) return true;
    fail();
    return false;
  }
};

// Dynamic scheduling: the producer warp takes units from a counter in the workspace's status
// area (units are numbered heaviest first) and hands them to the MMA and elementwise warps
// through a small ring; the last CTA to finish resets the counter for the next launch.
constexpr int kUnitSlots = 4;
constexpr int kUnitConsumers = 1 + kEw;
constexpr int kSchedWord = 16;  // int offset of the counter in the status area (+1: CTAs done)
struct UnitRing {
  uint64_t* full;   // [kUnitSlots]
  uint64_t* empty;  // [kUnitSlots]
  int* ring;        // [kUnitSlots]
  unsigned* sched;
  int n_units;
  // the producer's k-th unit (n_units once none is left)
  __device__ __forceinline__ bool take(const Waiter& W, uint32_t k, bool elected, int& u) const {
    const int slot = k % kUnitSlots;
    if (!W.all(&empty[slot], ((k / kUnitSlots) & 1) ^ 1)) return false;
    int v = 0;
    if (elected) {
      v = (int)atomicAdd(sched, 1u);
      if (v > n_units) v = n_units;
      ring[slot] = v;
      mbar_arrive(&full[slot]);
    }
    u = __shfl_sync(0xffffffffu, v, 0);
    return true;
  }
  // a consumer's k-th unit
  __device__ __forceinline__ bool next(const Waiter& W, uint32_t k, bool elected, int& u) const {
    const int slot = k % kUnitSlots;
    if (!W.all(&full[slot], (k / kUnitSlots) & 1)) return false;
    u = *reinterpret_cast<volatile int*>(&ring[slot]);
    __syncwarp();
    if (elected) mbar_arrive(&empty[slot]);
    return true;
  }
};
__device__ __forceinline__ void reset_scheduler(unsigned* sched) {
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(sched + 1, 1u) == gridDim.x - 1) {
      atomicExch(sched, 0u);
      atomicExch(sched + 1, 0u);
      __threadfence();
    }
  }
}

template <typename T>
__device__ __forceinline__ uint32_t pack16(float lo, float hi) {
  return std::is_same<T, __half>::value ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}
template <typename T>
__device__ __forceinline__ float low16(uint32_t w) {
  const uint16_t x = (uint16_t)(w & 0xFFFFu);
  return to_f32(*reinterpret_cast<const T*>(&x));
}
template <typename T>
__device__ __forceinline__ float high16(uint32_t w) {
  const uint16_t x = (uint16_t)(w >> 16);
  return to_f32(*reinterpret_cast<const T*>(&x));
}

// Bit e set for e in [a, b) (0 <= a, b <= 32 after clamping): the attended values of a chunk.
__device__ __forceinline__ uint32_t range_bits(int a, int b) {
  a = max(a, 0);
  b = min(b, 32);
  if (a >= b) return 0u;
  const uint32_t below_b = b >= 32 ? 0xffffffffu : (1u << b) - 1u;
  return below_b & ~((1u << a) - 1u);
}
// A pair (x0, x1) as its 16-bit high parts (one word) and the rounded remainders (one word).
template <typename T>
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack16<T>(x0, x1);
  float r0, r1;
  add2(r0, r1, x0, x1, -low16<T>(hi), -high16<T>(hi));
  lo = pack16<T>(r0, r1);
}
// 32 lanes x 16 consecutive 32-bit TMEM columns from registers.
// S-type MMA group: D[tmem] = A (128 x 128, K-major in smem) * B (128 x 128, K-major)^T
__device__ __forceinline__ void mma_kmajor(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk) {
    const uint32_t off = (kk / 4) * kRegion + (kk % 4) * 32;
    mma_ss(d, smem_desc_sw128(a + off, 16, 1024), smem_desc_sw128(b + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}
// PV-type MMA group: D[tmem] (+)= A (TMEM, 128 lanes x 128 values as 16-bit pairs, chunk-split
// high / low parts) * B (128 x 128 in smem, the K dimension along its rows: MN-major); `parts`
// 1 takes the high parts only
__device__ __forceinline__ void mma_tmem_a(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc, bool accumulate,
                                           int parts = 2) {
#pragma unroll
  for (int part = 0; part < 2; ++part) {
    if (part >= parts) break;
#pragma unroll
    for (int kk = 0; kk < kBlk / 16; ++kk) {
      // values [16 kk, 16 kk + 16) of part `part` sit in chunk kk / 2, 8 columns in
      const uint32_t acol = 32 * (kk / 2) + 16 * part + 8 * (kk % 2);
      const uint64_t bdesc = smem_desc_sw128(b + kk * 16 * 128, kRegion, 1024);
      mma_ts(d, a + acol, bdesc, idesc, (accumulate || part > 0 || kk > 0) ? 1u : 0u);
    }
  }
}

// ------------------------------------------------------------------------------- dK and dV
template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
bwd_kv_kernel(const __grid_constant__ Maps maps, const Problem P, const float* __restrict__ lse,
              const float* __restrict__ delta, T* __restrict__ dk, T* __restrict__ dv, int n_units) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* k_s = smem;                  // K tile of the unit
  uint8_t* v_s = k_s + kTile;           // V tile of the unit
  uint8_t* q_s = v_s + kTile;           // [2] Q tiles
  uint8_t* do_s = q_s + 2 * kTile;      // [2] dout tiles
  float* stage = reinterpret_cast<float*>(do_s + 2 * kTile);  // [2][256]
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage + 2 * 2 * kBlk);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + 1;
  uint64_t* qd_full = bars + 2;   // [2]
  uint64_t* qd_empty = bars + 4;  // [2]
  uint64_t* st_full = bars + 6;    // S^T of the step computed
  uint64_t* pt_full = bars + 7;    // w^T of the step written back (dV may start)
  uint64_t* dp_full = bars + 22;   // dP^T of the step computed
  uint64_t* dx_full = bars + 23;   // dx^T of the step written back (dK may start)
  uint64_t* acc_full = bars + 8;
  uint64_t* acc_free = bars + 9;
  uint64_t* drain = bars + 10;
  uint64_t* staged = bars + 11;   // lse / delta of the step staged by the 8 elementwise warps
  const UnitRing units{bars + 12, bars + 16, reinterpret_cast<int*>(bars + 20),
                       reinterpret_cast<unsigned*>(P.status) + kSchedWord, n_units};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const bool elected = lane == 0;
  if (threadIdx.x == 0) {
    mbar_init(staged, kEw);
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qd_full[s], 1);
      mbar_init(&qd_empty[s], 1);
    }
    mbar_init(st_full, 1);
    mbar_init(pt_full, kEw);
    mbar_init(dp_full, 1);
    mbar_init(dx_full, kEw);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, kEw);
    mbar_init(drain, 1);
    for (int x = 0; x < kUnitSlots; ++x) {
      mbar_init(&units.full[x], 1);
      mbar_init(&units.empty[x], kUnitConsumers);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && elected) {
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
    prefetch_tmap(&maps.dout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waiter W{abort_flag, P.status, P.wait_timeout_ns};
  // unit u: key tile u / (B Hkv) (the causal heaviest first), then batch, then kv head
  auto unit_of = [&](int u, int& b, int& kvh, int& kt) {
    kt = u / (P.B * P.Hkv);
    const int rem = u % (P.B * P.Hkv);
    b = rem / P.Hkv;
    kvh = rem % P.Hkv;
  };

  if (warp >= kEw) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kOtherRegs));

  if (warp == kProducerWarp) {
    [&] {
      uint32_t uc = 0, n = 0;
      for (uint32_t kq = 0;; ++kq) {
        int u;
        if (!units.take(W, kq, elected, u)) return;
        if (u >= n_units) break;
        int b, kvh, kt;
        unit_of(u, b, kvh, kt);
        const BatchInfo bi = resolve_batch(P, b);
        int qb, qe;
        qt_range_of(P, bi, kt, qb, qe);
        if (qe <= qb) continue;
        if (!W.all(kv_empty, (uc & 1) ^ 1)) return;
        if (elected) {
          mbar_arrive_expect_tx(kv_full, 2 * kTile);
          for (int r = 0; r < 2; ++r) {
            tma_load_4d(k_s + r * kRegion, &maps.k, kv_full, r * 64, kvh, kt * kBlk, b);
            tma_load_4d(v_s + r * kRegion, &maps.v, kv_full, r * 64, kvh, kt * kBlk, b);
          }
        }
        __syncwarp();
        ++uc;
        for (int hh = 0; hh < P.group; ++hh) {
          const int h = kvh * P.group + hh;
          for (int qt = qb; qt < qe; ++qt, ++n) {
            const int slot = n & 1;
            if (!W.all(&qd_empty[slot], ((n >> 1) & 1) ^ 1)) return;
            if (elected) {
              mbar_arrive_expect_tx(&qd_full[slot], 2 * kTile);
              for (int r = 0; r < 2; ++r) {
                tma_load_4d(q_s + slot * kTile + r * kRegion, &maps.q, &qd_full[slot], r * 64, h, qt * kBlk, b);
                tma_load_4d(do_s + slot * kTile + r * kRegion, &maps.dout, &qd_full[slot], r * 64, h, qt * kBlk, b);
              }
            }
            __syncwarp();
          }
        }
      }
    }();
  } else if (warp == kMmaWarp) {
    [&] {
      constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
      constexpr uint32_t idesc_s = instr_desc_f16(kBf16, false, false, kBlk, kBlk);
      constexpr uint32_t idesc_acc = instr_desc_f16(kBf16, false, true, kBlk, kD);
      const uint32_t st_t = tmem, dp_t = tmem + 128, dv_t = tmem + 256, dk_t = tmem + 384;
      const uint32_t k_a = smem_addr(k_s), v_a = smem_addr(v_s), q_a = smem_addr(q_s), do_a = smem_addr(do_s);
      uint32_t uc = 0, n = 0;
      for (uint32_t kq = 0;; ++kq) {
        int u;
        if (!units.next(W, kq, elected, u)) return;
        if (u >= n_units) break;
        int b, kvh, kt;
        unit_of(u, b, kvh, kt);
        const BatchInfo bi = resolve_batch(P, b);
        int qb, qe;
        qt_range_of(P, bi, kt, qb, qe);
        if (qe <= qb) continue;
        if (!W.all(kv_full, uc & 1)) return;
        const int steps = P.group * (qe - qb);
        // Issue order per step n: dV(n), S^T(n+1), dK(n), dP^T(n+1). The elementwise warps
        // publish w^T(n) before they read dP^T(n), so the exponentials of step n+1 run while
        // dK(n) and dP^T(n+1) are on the tensor pipe. S^T(n+1) overwrites w^T(n) after dV(n)
        // has read it, dP^T(n+1) overwrites dx^T(n) after dK(n): the pipe runs in order.
        if (!W.all(&qd_full[n & 1], (n >> 1) & 1)) return;
        tc_fence_after();
        if (elected) {
          mma_kmajor(st_t, k_a, q_a + (n & 1) * kTile, idesc_s);    // S^T = K Q^T
          mma_commit(st_full);
          mma_kmajor(dp_t, v_a, do_a + (n & 1) * kTile, idesc_s);   // dP^T = V dout^T
          mma_commit(dp_full);
        }
        __syncwarp();
        for (int s = 0; s < steps; ++s, ++n) {
          const int slot = n & 1, nslot = (n + 1) & 1;
          const bool more = s + 1 < steps;
          if (!W.all(pt_full, n & 1)) return;
          if (s == 0 && !W.all(acc_free, (uc & 1) ^ 1)) return;
          if (more && !W.all(&qd_full[nslot], ((n + 1) >> 1) & 1)) return;
          tc_fence_after();
          if (elected) {
            mma_tmem_a(dv_t, st_t, do_a + slot * kTile, idesc_acc, s > 0, 1);  // dV += w^T dout
            if (more) {
              mma_kmajor(st_t, k_a, q_a + nslot * kTile, idesc_s);
              mma_commit(st_full);
            }
          }
          __syncwarp();
          if (!W.all(dx_full, n & 1)) return;
          tc_fence_after();
          if (elected) {
            mma_tmem_a(dk_t, dp_t, q_a + slot * kTile, idesc_acc, s > 0);  // dK += dx^T Q
            mma_commit(&qd_empty[slot]);
            if (more) {
              mma_kmajor(dp_t, v_a, do_a + nslot * kTile, idesc_s);
              mma_commit(dp_full);
            }
          }
          __syncwarp();
        }
        if (elected) {
          mma_commit(acc_full);
          mma_commit(kv_empty);
        }
        __syncwarp();
        ++uc;
      }
    }();
  } else if (warp < kEw) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kEwRegs));
    [&] {
      const int quarter = warp % 4, half = warp / 4;
      const int r = quarter * 32 + lane;  // key row in the tile = TMEM lane
      const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
      const float sl2 = P.scale_log2;
      uint32_t uc = 0, n = 0;
      for (uint32_t kq = 0;; ++kq) {
        int u;
        if (!units.next(W, kq, elected, u)) return;
        if (u >= n_units) break;
        int b, kvh, kt;
        unit_of(u, b, kvh, kt);
        const BatchInfo bi = resolve_batch(P, b);
        int qb, qe;
        qt_range_of(P, bi, kt, qb, qe);
        const int j = kt * kBlk + r;  // key
        const long long krow = ((long long)b * P.Lk + j) * P.Hkv + kvh;
        T* drow = (half == 0 ? dk : dv) + krow * kD;
        if (qe <= qb) {
          // no query sees this key tile: dk = dv = 0
          if (j < P.Lk) {
#pragma unroll
            for (int c = 0; c < kD; c += 8) *reinterpret_cast<uint4*>(drow + c) = make_uint4(0u, 0u, 0u, 0u);
          }
          continue;
        }
        const int steps = P.group * (qe - qb);
        for (int s = 0; s < steps; ++s, ++n) {
          const int h = kvh * P.group + s / (qe - qb), qt = qb + s % (qe - qb);
          // lse and delta of the tile's 128 queries, staged in shared memory by the 256 threads
          float* st = stage + (n & 1) * 2 * kBlk;
          {
            const int t = threadIdx.x;  // 0..255
            const int i = qt * kBlk + (t & 127);
            const long long idx = ((long long)b * P.H + h) * P.Lq + i;
            float val = (t < 128) ? INFINITY : 0.f;
            if (i < P.Lq) val = (t < 128) ? lse[idx] * P.lse_in_mul : delta[idx];
            st[t] = val;
          }
          // every warp's values are in (a step's slot is rewritten two steps later, after every
          // warp has passed this point of the step in between)
          __syncwarp();
          if (elected) mbar_arrive(staged);
          if (!W.all(staged, n & 1)) return;
          if (!W.all(st_full, n & 1)) return;
          tc_fence_after();
          // key j attends queries [i_lo, i_hi): i < q_len, j < kv_len and (causal) j <= offset + i
          const int i_lo = P.causal != SDPA_CAUSAL_NONE ? j - bi.offset : 0;
          const int i_hi = j < bi.kv_len ? bi.q_len : 0;
          // phase 1: w^T from S^T, written back as 16-bit values (kept in fp32 for dx)
          float wv[2][32];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * half + cc;  // 32-query chunk
            const int q0 = qt * kBlk + 32 * c;
            const uint32_t keep = range_bits(i_lo - q0, i_hi - q0);
            uint32_t sv[32];
            tmem_ld32(lane_addr + 32 * c, sv);
            tmem_wait_ld();
            const float4* l4 = reinterpret_cast<const float4*>(st + 32 * c);
            uint32_t wo[16];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 L = l4[e / 4];
              const float lv[4] = {L.x, L.y, L.z, L.w};
#pragma unroll
              for (int y = 0; y < 4; y += 2) {
                const int f = e + y;
                float x0, x1;
                fma2(x0, x1, __uint_as_float(sv[f]), __uint_as_float(sv[f + 1]), sl2, sl2, -lv[y], -lv[y + 1]);
                wv[cc][f] = ((keep >> f) & 1u) ? ex2(x0) : 0.f;
                wv[cc][f + 1] = ((keep >> (f + 1)) & 1u) ? ex2(x1) : 0.f;
                wo[f / 2] = pack16<T>(wv[cc][f], wv[cc][f + 1]);
              }
            }
            tmem_st16(lane_addr + 32 * c, wo);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (elected) mbar_arrive(pt_full);
          // phase 2: dx^T = w^T (dP^T - delta), high and low parts over dP^T
          if (!W.all(dp_full, n & 1)) return;
          tc_fence_after();
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * half + cc;
            uint32_t dpv[32];
            tmem_ld32(lane_addr + 128 + 32 * c, dpv);
            tmem_wait_ld();
            const float4* d4 = reinterpret_cast<const float4*>(st + kBlk + 32 * c);
            uint32_t xo[32];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 Dl = d4[e / 4];
              const float dl[4] = {Dl.x, Dl.y, Dl.z, Dl.w};
#pragma unroll
              for (int y = 0; y < 4; y += 2) {
                const int f = e + y;
                float t0, t1, d0, d1;
                add2(t0, t1, __uint_as_float(dpv[f]), __uint_as_float(dpv[f + 1]), -dl[y], -dl[y + 1]);
                fma2(d0, d1, wv[cc][f], wv[cc][f + 1], t0, t1, 0.f, 0.f);  // dx = w (dp - delta)
                split_pair<T>(d0, d1, xo[f / 2], xo[16 + f / 2]);
              }
            }
            tmem_st32(lane_addr + 128 + 32 * c, xo);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (elected) mbar_arrive(dx_full);
        }
        // epilogue: dK (warps 0-3, times scale) or dV (warps 4-7), one row per thread
        if (!W.all(acc_full, uc & 1)) return;
        tc_fence_after();
        const float mulv = half == 0 ? P.scale : 1.f;
#pragma unroll 1
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t a[32];
          tmem_ld32(lane_addr + (half == 0 ? 384 : 256) + 32 * c, a);
          tmem_wait_ld();
          if (j < P.Lk) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint32_t wv[4];
#pragma unroll
              for (int z = 0; z < 4; ++z)
                wv[z] = pack16<T>(__uint_as_float(a[e + 2 * z]) * mulv, __uint_as_float(a[e + 2 * z + 1]) * mulv);
              *reinterpret_cast<uint4*>(drow + 32 * c + e) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (elected) mbar_arrive(acc_free);
        ++uc;
      }
    }();
  }
  if (warp == kMmaWarp) {
    if (elected) mma_commit(drain);
    __syncwarp();
    mbar_wait(drain, 0, P.wait_timeout_ns, nullptr);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  reset_scheduler(units.sched);
}

// ------------------------------------------------------------------------------- dQ and dscale
template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
bwd_q_kernel(const __grid_constant__ Maps maps, const Problem P, const float* __restrict__ lse,
             const float* __restrict__ delta, T* __restrict__ dq, float* __restrict__ dscale, int n_units) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem;               // Q tile of the unit
  uint8_t* do_s = q_s + kTile;       // dout tile of the unit
  uint8_t* k_s = do_s + kTile;       // [2] K tiles
  uint8_t* v_s = k_s + 2 * kTile;    // [2] V tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(v_s + 2 * kTile + 2 * 2 * kBlk * 4);
  uint64_t* qo_full = bars;
  uint64_t* qo_empty = bars + 1;
  uint64_t* kv_full = bars + 2;   // [2]
  uint64_t* kv_empty = bars + 4;  // [2]
  uint64_t* s_full = bars + 6;
  uint64_t* p_full = bars + 7;
  uint64_t* acc_full = bars + 8;
  uint64_t* acc_free = bars + 9;
  uint64_t* drain = bars + 10;
  const UnitRing units{bars + 12, bars + 16, reinterpret_cast<int*>(bars + 20),
                       reinterpret_cast<unsigned*>(P.status) + kSchedWord, n_units};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const bool elected = lane == 0;
  if (threadIdx.x == 0) {
    mbar_init(qo_full, 1);
    mbar_init(qo_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, kEw);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, kEw);
    mbar_init(drain, 1);
    for (int x = 0; x < kUnitSlots; ++x) {
      mbar_init(&units.full[x], 1);
      mbar_init(&units.empty[x], kUnitConsumers);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && elected) {
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
    prefetch_tmap(&maps.dout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Waiter W{abort_flag, P.status, P.wait_timeout_ns};
  const int nqt = (P.Lq + kBlk - 1) / kBlk;
  // unit u: query tile (nqt - 1 - u / (B H)) (the causal heaviest first), then batch, then head
  auto unit_of = [&](int u, int& b, int& h, int& qt) {
    qt = nqt - 1 - u / (P.B * P.H);
    const int rem = u % (P.B * P.H);
    b = rem / P.H;
    h = rem % P.H;
  };

  if (warp >= kEw) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kOtherRegs));

  if (warp == kProducerWarp) {
    [&] {
      uint32_t uc = 0, n = 0;
      for (uint32_t kq = 0;; ++kq) {
        int u;
        if (!units.take(W, kq, elected, u)) return;
        if (u >= n_units) break;
        int b, h, qt;
        unit_of(u, b, h, qt);
        const BatchInfo bi = resolve_batch(P, b);
        const int nk = kt_end_of(P, bi, qt);
        if (nk == 0) continue;
        const int kvh = h / P.group;
        if (!W.all(qo_empty, (uc & 1) ^ 1)) return;
        if (elected) {
          mbar_arrive_expect_tx(qo_full, 2 * kTile);
          for (int r = 0; r < 2; ++r) {
            tma_load_4d(q_s + r * kRegion, &maps.q, qo_full, r * 64, h, qt * kBlk, b);
            tma_load_4d(do_s + r * kRegion, &maps.dout, qo_full, r * 64, h, qt * kBlk, b);
          }
        }
        __syncwarp();
        ++uc;
        for (int kt = 0; kt < nk; ++kt, ++n) {
          const int slot = n & 1;
          if (!W.all(&kv_empty[slot], ((n >> 1) & 1) ^ 1)) return;
          if (elected) {
            mbar_arrive_expect_tx(&kv_full[slot], 2 * kTile);
            for (int r = 0; r < 2; ++r) {
              tma_load_4d(k_s + slot * kTile + r * kRegion, &maps.k, &kv_full[slot], r * 64, kvh, kt * kBlk, b);
              tma_load_4d(v_s + slot * kTile + r * kRegion, &maps.v, &kv_full[slot], r * 64, kvh, kt * kBlk, b);
            }
          }
          __syncwarp();
        }
      }
    }();
  } else if (warp == kMmaWarp) {
    [&] {
      constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
      constexpr uint32_t idesc_s = instr_desc_f16(kBf16, false, false, kBlk, kBlk);
      constexpr uint32_t idesc_acc = instr_desc_f16(kBf16, false, true, kBlk, kD);
      const uint32_t dp_t = tmem + 128, dq_t = tmem + 256;
      auto s_tm = [&](uint32_t x) { return tmem + ((x & 1) ? 384u : 0u); };  // S, two buffers
      const uint32_t q_a = smem_addr(q_s), do_a = smem_addr(do_s), k_a = smem_addr(k_s), v_a = smem_addr(v_s);
      uint32_t uc = 0, n = 0;
      for (uint32_t kq = 0;; ++kq) {
        int u;
        if (!units.next(W, kq, elected, u)) return;
        if (u >= n_units) break;
        int b, h, qt;
        unit_of(u, b, h, qt);
        const BatchInfo bi = resolve_batch(P, b);
        const int nk = kt_end_of(P, bi, qt);
        if (nk == 0) continue;
        if (!W.all(qo_full, uc & 1)) return;
        // Issue order: S(0), dP(0); then per key tile kt (ring position n): S(n+1) into the other
        // S buffer while the elementwise warps work on n, then (dx(n) written) dP(n+1) and
        // dQ(n). The elementwise phase of n+1 then waits for dP(n+1) only, and runs while
        // dQ(n) is on the tensor pipe. S(n+2) reuses the buffer of S(n) after dQ(n) read it.
        if (!W.all(&kv_full[n & 1], (n >> 1) & 1)) return;
        tc_fence_after();
        if (elected) {
          mma_kmajor(s_tm(n), q_a, k_a + (n & 1) * kTile, idesc_s);  // S = Q K^T
          mma_kmajor(dp_t, do_a, v_a + (n & 1) * kTile, idesc_s);    // dP = dout V^T
          mma_commit(s_full);
        }
        __syncwarp();
        for (int kt = 0; kt < nk; ++kt, ++n) {
          const int slot = n & 1, nslot = (n + 1) & 1;
          const bool more = kt + 1 < nk;
          if (more) {
            if (!W.all(&kv_full[nslot], ((n + 1) >> 1) & 1)) return;
            tc_fence_after();
            if (elected) mma_kmajor(s_tm(n + 1), q_a, k_a + nslot * kTile, idesc_s);
            __syncwarp();
          }
          if (!W.all(p_full, n & 1)) return;
          if (kt == 0 && !W.all(acc_free, (uc & 1) ^ 1)) return;
          tc_fence_after();
          if (elected) {
            if (more) {
              mma_kmajor(dp_t, do_a, v_a + nslot * kTile, idesc_s);
              mma_commit(s_full);
            }
            mma_tmem_a(dq_t, s_tm(n), k_a + slot * kTile, idesc_acc, kt > 0);  // dQ += dx K
            mma_commit(&kv_empty[slot]);
          }
          __syncwarp();
        }
        if (elected) {
          mma_commit(acc_full);
          mma_commit(qo_empty);
        }
        __syncwarp();
        ++uc;
      }
    }();
  } else if (warp < kEw) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kEwRegs));
    [&] {
      const int quarter = warp % 4, half = warp / 4;
      const int r = quarter * 32 + lane;  // query row in the tile = TMEM lane
      const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
      const float sl2 = P.scale_log2;
      float ds_acc0 = 0.f, ds_acc1 = 0.f;
      uint32_t uc = 0, n = 0;
      for (uint32_t kq = 0;; ++kq) {
        int u;
        if (!units.next(W, kq, elected, u)) return;
        if (u >= n_units) break;
        int b, h, qt;
        unit_of(u, b, h, qt);
        const BatchInfo bi = resolve_batch(P, b);
        const int nk = kt_end_of(P, bi, qt);
        const int i = qt * kBlk + r;
        T* qrow = dq + (((long long)b * P.Lq + i) * P.H + h) * kD + 64 * half;
        if (nk == 0) {
          if (i < P.Lq) {
#pragma unroll
            for (int c = 0; c < 64; c += 8) *reinterpret_cast<uint4*>(qrow + c) = make_uint4(0u, 0u, 0u, 0u);
          }
          continue;
        }
        const long long ridx = ((long long)b * P.H + h) * P.Lq + i;
        const float lse_i = i < P.Lq ? lse[ridx] * P.lse_in_mul : INFINITY;
        const float delta_i = i < P.Lq ? delta[ridx] : 0.f;
        long long lim = i < bi.q_len ? bi.kv_len : 0;
        if (P.causal != SDPA_CAUSAL_NONE) lim = min(lim, (long long)bi.offset + i + 1);
        const int j_lim = (int)max(lim, 0LL);  // keys j < j_lim are attended
        for (int kt = 0; kt < nk; ++kt, ++n) {
          if (!W.all(s_full, n & 1)) return;
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * half + cc;  // 32-key chunk
            const uint32_t keep = range_bits(0, j_lim - (kt * kBlk + 32 * c));
            uint32_t sv[32], dpv[32];
            const uint32_t scol = ((n & 1) ? 384u : 0u) + 32 * c;
            tmem_ld32(lane_addr + scol, sv);
            tmem_ld32(lane_addr + 128 + 32 * c, dpv);
            tmem_wait_ld();
            uint32_t xo[32];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float s0 = __uint_as_float(sv[e]), s1 = __uint_as_float(sv[e + 1]);
              float x0, x1, t0, t1, d0, d1;
              fma2(x0, x1, s0, s1, sl2, sl2, -lse_i, -lse_i);
              const float p0 = ((keep >> e) & 1u) ? ex2(x0) : 0.f;
              const float p1 = ((keep >> (e + 1)) & 1u) ? ex2(x1) : 0.f;
              add2(t0, t1, __uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1]), -delta_i, -delta_i);
              fma2(d0, d1, p0, p1, t0, t1, 0.f, 0.f);  // dx = w (dp - delta)
              fma2(ds_acc0, ds_acc1, d0, d1, s0, s1, ds_acc0, ds_acc1);
              split_pair<T>(d0, d1, xo[e / 2], xo[16 + e / 2]);
            }
            tmem_st32(lane_addr + scol, xo);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (elected) mbar_arrive(p_full);
        }
        // epilogue: this warp's 64 columns of dQ (times scale)
        if (!W.all(acc_full, uc & 1)) return;
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t a[32];
          tmem_ld32(lane_addr + 256 + 64 * half + 32 * cc, a);
          tmem_wait_ld();
          if (i < P.Lq) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint32_t wv[4];
#pragma unroll
              for (int z = 0; z < 4; ++z)
                wv[z] = pack16<T>(__uint_as_float(a[e + 2 * z]) * P.scale, __uint_as_float(a[e + 2 * z + 1]) * P.scale);
              *reinterpret_cast<uint4*>(qrow + 32 * cc + e) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (elected) mbar_arrive(acc_free);
        ++uc;
      }
      // dscale: this warp's sum, one atomic
      float ds_acc = ds_acc0 + ds_acc1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ds_acc += __shfl_xor_sync(0xffffffffu, ds_acc, o);
      if (elected && dscale && ds_acc != 0.f) atomicAdd(dscale, ds_acc);
    }();
  }
  if (warp == kMmaWarp) {
    if (elected) mma_commit(drain);
    __syncwarp();
    mbar_wait(drain, 0, P.wait_timeout_ns, nullptr);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  reset_scheduler(units.sched);
}

// delta = dout . out per (batch, head, query) row, [B][H][Lq]; half a warp per row, 16 bytes
// per lane
template <typename T>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const Problem P, const T* __restrict__ out,
                                                        const T* __restrict__ dout, float* __restrict__ delta) {
  const long long row = (long long)blockIdx.x * 16 + threadIdx.x / 16;  // (b, i, h), h fastest
  const int sub = threadIdx.x % 16;
  const bool live = row < (long long)P.B * P.Lq * P.H;
  float acc = 0.f;
  if (live) {
    const uint4 o = *reinterpret_cast<const uint4*>(out + row * kD + 8 * sub);
    const uint4 d = *reinterpret_cast<const uint4*>(dout + row * kD + 8 * sub);
    const uint32_t ow[4] = {o.x, o.y, o.z, o.w}, dw[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
    for (int z = 0; z < 4; ++z) acc += low16<T>(ow[z]) * low16<T>(dw[z]) + high16<T>(ow[z]) * high16<T>(dw[z]);
  }
#pragma unroll
  for (int x = 8; x > 0; x >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, x);
  if (live && sub == 0) {
    const int h = (int)(row % P.H);
    const long long bi_ = row / P.H;
    const int i = (int)(bi_ % P.Lq), b = (int)(bi_ / P.Lq);
    // a row with no key has a NaN output and takes no part: its weights are 0, and so is delta
    // (0 * (dp - NaN) would otherwise spread the NaN)
    delta[((long long)b * P.H + h) * P.Lq + i] = isnan(acc) ? 0.f : acc;
  }
}

template <typename K>
cudaError_t prepare(K kern) {
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
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    ready.fetch_or(bit, std::memory_order_acq_rel);
  }
  return cudaSuccess;
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

template <typename T>
cudaError_t launch_t(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                     const void* dout, void* dq, void* dk, void* dv, float* dscale, float* lse, float* delta,
                     cudaStream_t stream) {
  Maps maps{};
  if (!make_map(&maps.q, q, P.dtype, kD, P.H, P.Lq, P.B) || !make_map(&maps.dout, dout, P.dtype, kD, P.H, P.Lq, P.B) ||
      !make_map(&maps.k, k, P.dtype, kD, P.Hkv, P.Lk, P.B) || !make_map(&maps.v, v, P.dtype, kD, P.Hkv, P.Lk, P.B))
    return cudaErrorInvalidValue;
  const long long rows = (long long)P.B * P.Lq * P.H;
  bwd_delta_kernel<T><<<(unsigned)((rows + 15) / 16), 256, 0, stream>>>(P, (const T*)out, (const T*)dout, delta);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (dscale) {
    e = cudaMemsetAsync(dscale, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
  }
  e = prepare(bwd_kv_kernel<T>);
  if (e != cudaSuccess) return e;
  e = prepare(bwd_q_kernel<T>);
  if (e != cudaSuccess) return e;
  const int kv_units = P.B * P.Hkv * ((P.Lk + kBlk - 1) / kBlk);
  const int q_units = P.B * P.H * ((P.Lq + kBlk - 1) / kBlk);
  bwd_kv_kernel<T><<<std::min(kv_units, sm_count()), kThreads, kSmemBytes, stream>>>(maps, P, lse, delta, (T*)dk,
                                                                                     (T*)dv, kv_units);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_q_kernel<T><<<std::min(q_units, sm_count()), kThreads, kSmemBytes, stream>>>(maps, P, lse, delta, (T*)dq,
                                                                                   dscale, q_units);
  return cudaGetLastError();
}

}  // namespace bwd

bool backward_sm100_supported(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                              const void* dout, const void* dq, const void* dk, const void* dv) {
  if (P.dtype != SDPA_BF16 && P.dtype != SDPA_F16) return false;
  if (P.D != 128 || P.Dv != 128) return false;
  if (P.bias || P.mask || P.bcls || P.q_start) return false;
  if (P.B <= 0 || P.Lq <= 0 || P.Lk <= 0) return false;
  if (!(P.scale > 0.f)) return false;
  for (const void* p : {q, k, v, out, dout, dq, dk, dv})
    if (reinterpret_cast<uintptr_t>(p) % 16) return false;
  return (long long)P.B * P.H * ((P.Lq + 127) / 128) < (1LL << 30) &&
         (long long)P.B * P.Hkv * ((P.Lk + 127) / 128) < (1LL << 30);
}

cudaError_t launch_backward_sm100(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                                  const void* dout, void* dq, void* dk, void* dv, float* dscale, float* lse,
                                  float* delta, cudaStream_t stream) {
  if (P.dtype == SDPA_BF16)
    return bwd::launch_t<__nv_bfloat16>(P, q, k, v, out, dout, dq, dk, dv, dscale, lse, delta, stream);
  return bwd::launch_t<__half>(P, q, k, v, out, dout, dq, dk, dv, dscale, lse, delta, stream);
}

}  // namespace sdpa
