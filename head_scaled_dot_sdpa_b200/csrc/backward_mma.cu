// The gradient of the fused implementation on the tensor cores (Flux.jl page "Neural Network
// primitives from NNlib.jl", entry scaled_dot_product_attention, paragraph "Fused
// implementation": a gradient with respect to query, key, value and scale that recomputes the
// weights tile by tile; a query whose output is NaN takes no part).
//
// bf16 / fp16 with head_dim = v_head_dim = 64 or 128, on mma.sync m16n8k16 (fp32 accumulate):
//  - bwd_dq_mma: one CTA per (64-query tile, head, batch), 4 warps of 16 query rows. Pass 1
//    walks the key tiles for the row log-sum-exp (S = Q K^T). Pass 2 walks them again:
//    S and dP = dout V^T, w = 2^(S scale log2e - lse), dx = w (dP - delta) with
//    delta = dout . out, dq += dx K, and dscale += dx (q . k). It writes dq, and lse and delta
//    for the second kernel.
//  - bwd_dkdv_mma: one CTA per (64-key tile, kv head, batch), 4 warps of 16 keys. It walks the
//    32-query tiles of every query head of the group, computing S^T = K Q^T and
//    dP^T = V dout^T, then dv += w^T dout and dk += dx^T Q. So each dk / dv row is written
//    once, without atomics.
// Tiles are staged in shared memory with cp.async (16-byte chunks, rows XOR-swizzled by
// chunk) and read with ldmatrix. The weight and dx accumulators are reused as A operands, each
// split into a 16-bit hi and lo part (two MMAs), so the gradient's products keep fp32 accuracy.
#include "mma_tiles.cuh"

namespace sdpa {
namespace {

using namespace tiles;

constexpr int kQRows = 64;   // dq kernel: query rows per CTA
constexpr int kKeys = 64;    // keys per tile (both kernels)
constexpr int kQTile = 32;   // dk/dv kernel: query rows per tile

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
bwd_dq_mma(Problem P, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
           const T* __restrict__ out, const T* __restrict__ dout, float* __restrict__ lse_ws,
           float* __restrict__ delta_ws, T* __restrict__ dq, float* dscale) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float delta_s[kQRows];
  __shared__ float red[kWarps];
  constexpr int kTileBytes = kQRows * D * 2;
  const Tile<D> tq{su32(smem)}, tdo{su32(smem + kTileBytes)};
  const Tile<D> tk[2] = {{su32(smem + 2 * kTileBytes)}, {su32(smem + 3 * kTileBytes)}};
  const Tile<D> tv[2] = {{su32(smem + 4 * kTileBytes)}, {su32(smem + 5 * kTileBytes)}};
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, gq = lane / 4, tq4 = lane % 4;
  const int h = blockIdx.y, b = blockIdx.z, i0 = blockIdx.x * kQRows;
  const BatchInfo bi = resolve_batch(P, b);
  if (i0 >= bi.q_rows) return;
  const int g = h / P.group;
  const long long qstride = (long long)P.H * D, kstride = (long long)P.Hkv * D;
  const T* qb = q + (bi.q0 * P.H + h) * D;
  const T* dob = dout + (bi.q0 * P.H + h) * D;
  const T* kb = k + (bi.k0 * P.Hkv + g) * D;
  const T* vb = v + (bi.k0 * P.Hkv + g) * D;
  const int qvalid = min(kQRows, bi.q_len - i0);  // rows that attend (rows past q_len: dq = 0)
  float ds_acc = 0.f;
  float acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  const int rl = warp * 16 + gq, rh = rl + 8;  // this thread's two rows in the tile
  const int il = i0 + rl, ih = i0 + rh;
  float lse_l = INFINITY, lse_h = INFINITY;
  if (qvalid > 0) {
    load_rows<T, D>(tq, qb, i0, qvalid, kQRows, qstride);
    load_rows<T, D>(tdo, dob, i0, qvalid, kQRows, qstride);
    cp_commit();
    // delta = dout . out per row
    for (int rr = 0; rr < 16; ++rr) {
      const int r = warp * 16 + rr, i = i0 + r;
      float d = 0.f;
      if (r < qvalid) {
        const long long o = ((bi.q0 + i) * P.H + h) * D;
        for (int e = lane; e < D; e += 32) d = fmaf(to_f32(dout[o + e]), to_f32(out[o + e]), d);
      }
#pragma unroll
      for (int s = 16; s > 0; s >>= 1) d += __shfl_xor_sync(0xffffffffu, d, s);
      if (lane == 0) delta_s[r] = d;
    }
    __syncwarp();  // each warp reads only its own rows' delta
    // keys any row of the tile may attend
    long long jend = bi.kv_len;
    if (P.causal != SDPA_CAUSAL_NONE) jend = min(jend, (long long)bi.offset + i0 + qvalid);
    const int nkt = jend > 0 ? (int)((jend + kKeys - 1) / kKeys) : 0;
    const float c2 = P.scale * kLog2e;

    // pass 1: row max and sum of 2^(S c2) over the attended keys
    float m_l = -INFINITY, m_h = -INFINITY, l_l = 0.f, l_h = 0.f;
    if (nkt > 0) {
      load_rows<T, D>(tk[0], kb, 0, min(kKeys, P.Lk), kKeys, kstride);
      cp_commit();
    }
    for (int t = 0; t < nkt; ++t) {
      if (t + 1 < nkt) {
        load_rows<T, D>(tk[(t + 1) & 1], kb, (long long)(t + 1) * kKeys, min(kKeys, P.Lk - (t + 1) * kKeys), kKeys,
                        kstride);
        cp_commit();
        cp_wait<1>();
      } else {
        cp_wait<0>();
      }
      __syncthreads();
      float s[kKeys / 8][4];
#pragma unroll
      for (int n = 0; n < kKeys / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        frag_a(tq, warp * 16, kk * 16, a);
#pragma unroll
        for (int np = 0; np < kKeys / 16; ++np) {
          uint32_t bb[4];
          frag_b_nk(tk[t & 1], np * 16, kk * 16, bb);
          mma<T>(s[2 * np], a, bb[0], bb[1]);
          mma<T>(s[2 * np + 1], a, bb[2], bb[3]);
        }
      }
#pragma unroll
      for (int n = 0; n < kKeys / 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = t * kKeys + n * 8 + 2 * tq4 + (e & 1);
          const int i = (e < 2) ? il : ih;
          const bool ok = i < bi.q_len && allowed(P, bi, b, h, i, j);
          const float x = ok ? s[n][e] * c2 : -INFINITY;
          float& m = (e < 2) ? m_l : m_h;
          float& l = (e < 2) ? l_l : l_h;
          if (x != -INFINITY) {
            if (x > m) {
              l = l * exp2f(m - x) + 1.f;
              m = x;
            } else {
              l += exp2f(x - m);
            }
          }
        }
      }
      __syncthreads();  // the tile is free for the load two steps ahead
    }
    // merge the four threads of each row
    {
      const float M_l = quad_max(m_l), M_h = quad_max(m_h);
      const float sl = quad_sum(m_l == -INFINITY ? 0.f : l_l * exp2f(m_l - M_l));
      const float sh = quad_sum(m_h == -INFINITY ? 0.f : l_h * exp2f(m_h - M_h));
      lse_l = sl > 0.f ? M_l + log2f(sl) : INFINITY;  // no attended key: no part in the gradient
      lse_h = sh > 0.f ? M_h + log2f(sh) : INFINITY;
    }
    const float dl_l = rl < qvalid ? delta_s[rl] : 0.f, dl_h = rh < qvalid ? delta_s[rh] : 0.f;

    // pass 2: dq += dx K, with dx = w (dP - delta)
    if (nkt > 0) {
      load_rows<T, D>(tk[0], kb, 0, min(kKeys, P.Lk), kKeys, kstride);
      load_rows<T, D>(tv[0], vb, 0, min(kKeys, P.Lk), kKeys, kstride);
      cp_commit();
    }
    for (int t = 0; t < nkt; ++t) {
      if (t + 1 < nkt) {
        const long long r0 = (long long)(t + 1) * kKeys;
        const int valid = min(kKeys, P.Lk - (t + 1) * kKeys);
        load_rows<T, D>(tk[(t + 1) & 1], kb, r0, valid, kKeys, kstride);
        load_rows<T, D>(tv[(t + 1) & 1], vb, r0, valid, kKeys, kstride);
        cp_commit();
        cp_wait<1>();
      } else {
        cp_wait<0>();
      }
      __syncthreads();
      float s[kKeys / 8][4], dp[kKeys / 8][4];
#pragma unroll
      for (int n = 0; n < kKeys / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4], ad[4];
        frag_a(tq, warp * 16, kk * 16, a);
        frag_a(tdo, warp * 16, kk * 16, ad);
#pragma unroll
        for (int np = 0; np < kKeys / 16; ++np) {
          uint32_t bb[4], bv[4];
          frag_b_nk(tk[t & 1], np * 16, kk * 16, bb);
          frag_b_nk(tv[t & 1], np * 16, kk * 16, bv);
          mma<T>(s[2 * np], a, bb[0], bb[1]);
          mma<T>(s[2 * np + 1], a, bb[2], bb[3]);
          mma<T>(dp[2 * np], ad, bv[0], bv[1]);
          mma<T>(dp[2 * np + 1], ad, bv[2], bv[3]);
        }
      }
      // dx in place of dp
#pragma unroll
      for (int n = 0; n < kKeys / 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = t * kKeys + n * 8 + 2 * tq4 + (e & 1);
          const int i = (e < 2) ? il : ih;
          const bool ok = i < bi.q_len && allowed(P, bi, b, h, i, j);
          // only attended pairs: a row with no key has a NaN delta, and 0 * NaN is NaN
          const float w = ok ? exp2f(s[n][e] * c2 - ((e < 2) ? lse_l : lse_h)) : 0.f;
          const float dx = ok ? w * (dp[n][e] - ((e < 2) ? dl_l : dl_h)) : 0.f;
          ds_acc = fmaf(dx, s[n][e], ds_acc);
          dp[n][e] = dx;
        }
      }
#pragma unroll
      for (int ks = 0; ks < kKeys / 16; ++ks) {
        uint32_t a[4], al[4];
        split2<T>(dp[2 * ks][0], dp[2 * ks][1], a[0], al[0]);
        split2<T>(dp[2 * ks][2], dp[2 * ks][3], a[1], al[1]);
        split2<T>(dp[2 * ks + 1][0], dp[2 * ks + 1][1], a[2], al[2]);
        split2<T>(dp[2 * ks + 1][2], dp[2 * ks + 1][3], a[3], al[3]);
#pragma unroll
        for (int nd = 0; nd < D / 16; ++nd) {
          uint32_t bb[4];
          frag_b_kn(tk[t & 1], ks * 16, nd * 16, bb);
          mma<T>(acc[2 * nd], a, bb[0], bb[1]);
          mma<T>(acc[2 * nd + 1], a, bb[2], bb[3]);
          mma<T>(acc[2 * nd], al, bb[0], bb[1]);
          mma<T>(acc[2 * nd + 1], al, bb[2], bb[3]);
        }
      }
      __syncthreads();
    }
    cp_wait<0>();  // with no key tile the Q / dout loads are still in flight
    __syncthreads();
  }
  // dq (zero for rows past q_lengths or with no key), lse and delta for the dk/dv kernel
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = half ? rh : rl, i = i0 + r;
    if (i >= bi.q_rows) continue;
    const long long row = (bi.q0 + i) * P.H + h;
    T* dst = dq + row * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const float x0 = acc[n][2 * half] * P.scale, x1 = acc[n][2 * half + 1] * P.scale;
      *reinterpret_cast<uint32_t*>(dst + n * 8 + 2 * tq4) = pk<T>(x0, x1);
    }
    if (tq4 == 0) {
      const float L = (r < qvalid) ? (half ? lse_h : lse_l) : INFINITY;
      lse_ws[row] = L;
      delta_ws[row] = L != INFINITY ? delta_s[r] : 0.f;  // rows with no key: NaN out, no part
    }
  }
  // dscale: sum of dx (q . k), one atomic per CTA
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) ds_acc += __shfl_xor_sync(0xffffffffu, ds_acc, s);
  if (lane == 0) red[warp] = ds_acc;
  __syncthreads();
  if (dscale && threadIdx.x == 0) {
    const float t = red[0] + red[1] + red[2] + red[3];
    if (t != 0.f) atomicAdd(dscale, t);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
bwd_dkdv_mma(Problem P, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
             const T* __restrict__ dout, const float* __restrict__ lse_ws, const float* __restrict__ delta_ws,
             T* __restrict__ dk, T* __restrict__ dv) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float lse_s[2][kQTile], delta_s[2][kQTile];
  constexpr int kKBytes = kKeys * D * 2, kQBytes = kQTile * D * 2;
  const Tile<D> tk{su32(smem)}, tv{su32(smem + kKBytes)};
  const Tile<D> tq[2] = {{su32(smem + 2 * kKBytes)}, {su32(smem + 2 * kKBytes + kQBytes)}};
  const Tile<D> tdo[2] = {{su32(smem + 2 * kKBytes + 2 * kQBytes)}, {su32(smem + 2 * kKBytes + 3 * kQBytes)}};
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, gq = lane / 4, tq4 = lane % 4;
  const int g = blockIdx.y, b = blockIdx.z, j0 = blockIdx.x * kKeys;
  if (j0 >= P.Lk) return;
  const BatchInfo bi = resolve_batch(P, b);
  const long long qstride = (long long)P.H * D, kstride = (long long)P.Hkv * D;
  float ak[D / 8][4], av[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) ak[n][e] = av[n][e] = 0.f;
  const int rl = warp * 16 + gq, rh = rl + 8;  // this thread's two keys in the tile
  const int jl = j0 + rl, jh = j0 + rh;
  if (j0 < bi.kv_len) {
    const T* kb = k + (bi.k0 * P.Hkv + g) * D;
    const T* vb = v + (bi.k0 * P.Hkv + g) * D;
    load_rows<T, D>(tk, kb, j0, min(kKeys, P.Lk - j0), kKeys, kstride);
    load_rows<T, D>(tv, vb, j0, min(kKeys, P.Lk - j0), kKeys, kstride);
    cp_commit();
    // query tiles that may see a key of this tile: i >= j0 - offset (causal), i < q_len
    long long first = 0;
    if (P.causal != SDPA_CAUSAL_NONE) first = max(0LL, (long long)j0 - bi.offset);
    if (first > bi.q_len) first = bi.q_len;
    const int it0 = ((int)first / kQTile) * kQTile;
    const int ntiles_h = bi.q_len > it0 ? (bi.q_len - it0 + kQTile - 1) / kQTile : 0;
    const int nsteps = ntiles_h * P.group;
    const float c2 = P.scale * kLog2e;
    auto stage = [&](int step, int buf) {
      const int h = g * P.group + step / ntiles_h;
      const int ib = it0 + (step % ntiles_h) * kQTile;
      const int valid = min(kQTile, bi.q_len - ib);
      const T* qb = q + (bi.q0 * P.H + h) * D;
      const T* dob = dout + (bi.q0 * P.H + h) * D;
      load_rows<T, D>(tq[buf], qb, ib, valid, kQTile, qstride);
      load_rows<T, D>(tdo[buf], dob, ib, valid, kQTile, qstride);
      if (threadIdx.x < kQTile) {
        const int i = ib + threadIdx.x;
        const long long row = (bi.q0 + i) * P.H + h;
        lse_s[buf][threadIdx.x] = i < bi.q_len ? lse_ws[row] : INFINITY;
        delta_s[buf][threadIdx.x] = i < bi.q_len ? delta_ws[row] : 0.f;
      }
    };
    if (nsteps > 0) {
      stage(0, 0);
      cp_commit();
    }
    for (int st = 0; st < nsteps; ++st) {
      const int buf = st & 1;
      if (st + 1 < nsteps) {
        stage(st + 1, buf ^ 1);
        cp_commit();
        cp_wait<1>();
      } else {
        cp_wait<0>();
      }
      __syncthreads();
      const int h = g * P.group + st / ntiles_h;
      const int ib = it0 + (st % ntiles_h) * kQTile;
      float s[kQTile / 8][4], dp[kQTile / 8][4];
#pragma unroll
      for (int n = 0; n < kQTile / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
      // S^T = K Q^T and dP^T = V dout^T for this warp's 16 keys x 32 queries
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4], avv[4];
        frag_a(tk, warp * 16, kk * 16, a);
        frag_a(tv, warp * 16, kk * 16, avv);
#pragma unroll
        for (int np = 0; np < kQTile / 16; ++np) {
          uint32_t bq[4], bd[4];
          frag_b_nk(tq[buf], np * 16, kk * 16, bq);
          frag_b_nk(tdo[buf], np * 16, kk * 16, bd);
          mma<T>(s[2 * np], a, bq[0], bq[1]);
          mma<T>(s[2 * np + 1], a, bq[2], bq[3]);
          mma<T>(dp[2 * np], avv, bd[0], bd[1]);
          mma<T>(dp[2 * np + 1], avv, bd[2], bd[3]);
        }
      }
      // w^T in s, dx^T in dp
#pragma unroll
      for (int n = 0; n < kQTile / 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = n * 8 + 2 * tq4 + (e & 1);
          const int i = ib + c, j = (e < 2) ? jl : jh;
          const bool ok = i < bi.q_len && j < P.Lk && allowed(P, bi, b, h, i, j);
          const float w = ok ? exp2f(s[n][e] * c2 - lse_s[buf][c]) : 0.f;
          dp[n][e] = ok ? w * (dp[n][e] - delta_s[buf][c]) : 0.f;
          s[n][e] = w;
        }
      }
      // dv += w^T dout, dk += dx^T Q (k dimension: the 32 queries)
#pragma unroll
      for (int ks = 0; ks < kQTile / 16; ++ks) {
        uint32_t a[4], al[4];
        split2<T>(s[2 * ks][0], s[2 * ks][1], a[0], al[0]);
        split2<T>(s[2 * ks][2], s[2 * ks][3], a[1], al[1]);
        split2<T>(s[2 * ks + 1][0], s[2 * ks + 1][1], a[2], al[2]);
        split2<T>(s[2 * ks + 1][2], s[2 * ks + 1][3], a[3], al[3]);
#pragma unroll
        for (int nd = 0; nd < D / 16; ++nd) {
          uint32_t bd[4];
          frag_b_kn(tdo[buf], ks * 16, nd * 16, bd);
          mma<T>(av[2 * nd], a, bd[0], bd[1]);
          mma<T>(av[2 * nd + 1], a, bd[2], bd[3]);
          mma<T>(av[2 * nd], al, bd[0], bd[1]);
          mma<T>(av[2 * nd + 1], al, bd[2], bd[3]);
        }
        split2<T>(dp[2 * ks][0], dp[2 * ks][1], a[0], al[0]);
        split2<T>(dp[2 * ks][2], dp[2 * ks][3], a[1], al[1]);
        split2<T>(dp[2 * ks + 1][0], dp[2 * ks + 1][1], a[2], al[2]);
        split2<T>(dp[2 * ks + 1][2], dp[2 * ks + 1][3], a[3], al[3]);
#pragma unroll
        for (int nd = 0; nd < D / 16; ++nd) {
          uint32_t bq[4];
          frag_b_kn(tq[buf], ks * 16, nd * 16, bq);
          mma<T>(ak[2 * nd], a, bq[0], bq[1]);
          mma<T>(ak[2 * nd + 1], a, bq[2], bq[3]);
          mma<T>(ak[2 * nd], al, bq[0], bq[1]);
          mma<T>(ak[2 * nd + 1], al, bq[2], bq[3]);
        }
      }
      __syncthreads();  // buffers are refilled two steps ahead
    }
    cp_wait<0>();
  }
  // a key row gets one write of dk and dv (zero for keys no query attends)
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int j = half ? jh : jl;
    if (j >= P.Lk) continue;
    const long long row = (bi.k0 + j) * P.Hkv + g;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      *reinterpret_cast<uint32_t*>(dk + row * D + n * 8 + 2 * tq4) =
          pk<T>(ak[n][2 * half] * P.scale, ak[n][2 * half + 1] * P.scale);
      *reinterpret_cast<uint32_t*>(dv + row * D + n * 8 + 2 * tq4) = pk<T>(av[n][2 * half], av[n][2 * half + 1]);
    }
  }
}

template <typename T, int D>
cudaError_t launch_td(const Problem& P, const void* q, const void* k, const void* v, const void* out, const void* dout,
                      void* dq, void* dk, void* dv, float* dscale, float* lse, float* delta, cudaStream_t stream) {
  const size_t smem_dq = (size_t)6 * kQRows * D * 2;
  const size_t smem_kv = (size_t)2 * kKeys * D * 2 + (size_t)4 * kQTile * D * 2;
  // set on every call: the attribute belongs to the current device's context
  cudaError_t ea = cudaFuncSetAttribute(bwd_dq_mma<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_dq);
  if (ea == cudaSuccess)
    ea = cudaFuncSetAttribute(bwd_dkdv_mma<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_kv);
  if (ea != cudaSuccess) return ea;
  if (dscale) {
    cudaError_t e = cudaMemsetAsync(dscale, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
  }
  if (P.B > 0 && P.Lq > 0) {
    const dim3 grid((unsigned)((P.Lq + kQRows - 1) / kQRows), (unsigned)P.H, (unsigned)P.B);
    bwd_dq_mma<T, D><<<grid, kWarps * 32, smem_dq, stream>>>(P, (const T*)q, (const T*)k, (const T*)v,
                                                              (const T*)out, (const T*)dout, lse, delta, (T*)dq,
                                                              dscale);
  }
  if (P.B > 0 && P.Lk > 0) {
    const dim3 grid((unsigned)((P.Lk + kKeys - 1) / kKeys), (unsigned)P.Hkv, (unsigned)P.B);
    bwd_dkdv_mma<T, D><<<grid, kWarps * 32, smem_kv, stream>>>(P, (const T*)q, (const T*)k, (const T*)v,
                                                                (const T*)dout, lse, delta, (T*)dk, (T*)dv);
  }
  return cudaGetLastError();
}

}  // namespace

bool backward_mma_supported(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                            const void* dout) {
  if (P.dtype != SDPA_BF16 && P.dtype != SDPA_F16) return false;
  if (P.D != P.Dv || (P.D != 64 && P.D != 128)) return false;
  if (P.q_start) return false;
  if (P.H > 65535 || P.Hkv > 65535 || P.B > 65535) return false;
  for (const void* p : {q, k, v, out, dout})
    if (reinterpret_cast<uintptr_t>(p) % 16) return false;
  return true;
}

cudaError_t launch_backward_mma(const Problem& P, const void* q, const void* k, const void* v, const void* out,
                                const void* dout, void* dq, void* dk, void* dv, float* dscale, void* ws,
                                cudaStream_t stream) {
  const long long rows = (long long)P.B * P.Lq * P.H;
  float* lse = static_cast<float*>(ws);
  float* delta = lse + ((rows + 63) / 64) * 64;
  if (P.dtype == SDPA_BF16)
    return P.D == 128 ? launch_td<__nv_bfloat16, 128>(P, q, k, v, out, dout, dq, dk, dv, dscale, lse, delta, stream)
                      : launch_td<__nv_bfloat16, 64>(P, q, k, v, out, dout, dq, dk, dv, dscale, lse, delta, stream);
  return P.D == 128 ? launch_td<__half, 128>(P, q, k, v, out, dout, dq, dk, dv, dscale, lse, delta, stream)
                    : launch_td<__half, 64>(P, q, k, v, out, dout, dq, dk, dv, dscale, lse, delta, stream);
}

}  // namespace sdpa
