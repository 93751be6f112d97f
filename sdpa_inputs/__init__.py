"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This module holds the workload recipes only: shapes, random draws and the construction of
bias and mask arrays. It holds none of the attention arithmetic, and imports neither the
CUDA package nor the oracle.

Layout: row-major (batch, seq_len, nheads, head_dim) for q/k/v, which is the column-major
(head_dim, nheads, seq_len, batch) of the Flux.jl page "Neural Network primitives from
NNlib.jl" (scaled_dot_product_attention). Bias and mask are row-major (nheads, q_len,
kv_len), i.e. the page's (kv_len, q_len, nheads) broadcast over the batch.

Random numbers: numpy's PCG64 seeded per workload for q/k/v, lengths, bias noise and block
classes; the partial-block mask bits use a counter-based generator (the 64-bit finalizer of
Appleby's MurmurHash3, "fmix64"), written once for numpy (host rows) and once for torch
(whole mask on the device), so either side can produce any part of the mask on its own.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    q_len: int
    kv_len: int
    nheads: int
    nkvheads: int
    head_dim: int
    dtype: str
    causal: object = False          # False, True or "bottom_right"
    seed: int = 0
    # decode only
    capacity: int = 0
    kv_len_min: int = 0
    kv_len_max: int = 0
    # bias only
    bias: bool = False
    bias_noise_std: float = 0.0
    # block-sparse mask only
    block: int = 0
    p_empty: float = 0.0
    p_full: float = 0.0
    p_partial: float = 0.0
    # packed sequences only: sequence lengths drawn uniformly from [seg_min, seg_max]
    seg_min: int = 0
    seg_max: int = 0


# The five workloads of the benchmark plan, with the sizes they are quoted on.
TINY_FP32 = Workload("tiny_fp32_d16_h2_l8", batch=1, q_len=8, kv_len=8, nheads=2, nkvheads=2,
                     head_dim=16, dtype="f32", causal=False, seed=1)
CAUSAL_GQA_PREFILL = Workload("causal_gqa_prefill_bf16_b4_h32kv8_d128_l2048", batch=4,
                              q_len=2048, kv_len=2048, nheads=32, nkvheads=8, head_dim=128,
                              dtype="bf16", causal=True, seed=2)
KV_CACHE_DECODE = Workload("kv_cache_decode_bf16_b64_h32kv8_d128_cap8192", batch=64, q_len=1,
                           kv_len=8192, nheads=32, nkvheads=8, head_dim=128, dtype="bf16",
                           causal="bottom_right", seed=3, capacity=8192, kv_len_min=512,
                           kv_len_max=8192)
ALIBI_T5_BIAS = Workload("alibi_t5_bias_fp16_b2_h16_d64_l4096", batch=2, q_len=4096,
                         kv_len=4096, nheads=16, nkvheads=16, head_dim=64, dtype="f16",
                         causal=True, seed=4, bias=True, bias_noise_std=0.5)
BLOCK_SPARSE = Workload("block_sparse_mask_bf16_b1_h16_d128_l16384", batch=1, q_len=16384,
                        kv_len=16384, nheads=16, nkvheads=16, head_dim=128, dtype="bf16",
                        causal=False, seed=5, block=128, p_empty=0.5, p_full=0.3,
                        p_partial=0.2)

# Documents of 64 to 4096 positions packed into 65536 positions (keywords q_segments /
# kv_segments; the heads and head size of the causal GQA prefill). q_len / kv_len are the
# packed totals; batch is unused.
PACKED_DOCS = Workload("packed_docs_causal_gqa_bf16_h32kv8_d128_t65536", batch=1, q_len=65536,
                       kv_len=65536, nheads=32, nkvheads=8, head_dim=128, dtype="bf16",
                       causal=True, seed=6, seg_min=64, seg_max=4096)

ALL = (TINY_FP32, CAUSAL_GQA_PREFILL, KV_CACHE_DECODE, ALIBI_T5_BIAS, BLOCK_SPARSE, PACKED_DOCS)


def scaled(w: Workload, **changes) -> Workload:
    """The same recipe at other sizes (smaller parity cases)."""
    return dataclasses.replace(w, **changes)


def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal(rng: np.random.Generator, shape, dtype: str) -> torch.Tensor:
    """i.i.d. N(0,1) drawn in float32, rounded (to nearest even) to `dtype`; CPU tensor."""
    x = rng.standard_normal(size=shape, dtype=np.float32)
    return torch.from_numpy(x).to(DTYPES[dtype])


def qkv(w: Workload, rng: np.random.Generator | None = None):
    """q (B, Lq, H, d), k and v (B, Lk, Hkv, d) in the workload dtype (CPU tensors)."""
    rng = rng or rng_for(w.seed)
    q = normal(rng, (w.batch, w.q_len, w.nheads, w.head_dim), w.dtype)
    k = normal(rng, (w.batch, w.kv_len, w.nkvheads, w.head_dim), w.dtype)
    v = normal(rng, (w.batch, w.kv_len, w.nkvheads, w.head_dim), w.dtype)
    return q, k, v


def decode_inputs(w: Workload):
    """KV-cache decode step: q (B, 1, H, d); caches (B, capacity, Hkv, d) filled with N(0,1)
    everywhere (also past each sequence's length); new k/v rows (B, 1, Hkv, d); and
    kv_lengths[b] ~ uniform integer in [kv_len_min, kv_len_max]. The new token is written at
    index kv_lengths[b] - 1, so that after the write the sequence has kv_lengths[b] keys."""
    rng = rng_for(w.seed)
    kv_lengths = rng.integers(w.kv_len_min, w.kv_len_max, size=w.batch, endpoint=True)
    q = normal(rng, (w.batch, w.q_len, w.nheads, w.head_dim), w.dtype)
    k_new = normal(rng, (w.batch, w.q_len, w.nkvheads, w.head_dim), w.dtype)
    v_new = normal(rng, (w.batch, w.q_len, w.nkvheads, w.head_dim), w.dtype)
    shape = (w.batch, w.capacity, w.nkvheads, w.head_dim)
    k_cache = normal(rng, shape, w.dtype)
    v_cache = normal(rng, shape, w.dtype)
    index = (kv_lengths - w.q_len).astype(np.int32)
    return dict(q=q, k_new=k_new, v_new=v_new, k_cache=k_cache, v_cache=v_cache,
                index=torch.from_numpy(index), kv_lengths=torch.from_numpy(kv_lengths.astype(np.int32)))


def alibi_t5_bias(w: Workload) -> torch.Tensor:
    """Bias of row-major shape (H, Lq, Lk): the ALiBi slope of head h (h = 1..H),
    2^(-8h/H), times (j - i), plus T5-style N(0, std^2) noise, drawn in float32 and rounded
    to the workload dtype. Drawn from its own stream (seed + 1000)."""
    rng = rng_for(w.seed + 1000)
    H, Lq, Lk = w.nheads, w.q_len, w.kv_len
    out = torch.empty((H, Lq, Lk), dtype=DTYPES[w.dtype])
    rel = (np.arange(Lk, dtype=np.float32)[None, :] - np.arange(Lq, dtype=np.float32)[:, None])
    for h in range(H):
        slope = np.float32(2.0 ** (-8.0 * (h + 1) / H))
        noise = rng.standard_normal(size=(Lq, Lk), dtype=np.float32) * np.float32(w.bias_noise_std)
        out[h] = torch.from_numpy(slope * rel + noise).to(out.dtype)
    return out


# ---- block-sparse boolean mask -------------------------------------------------------------

_C1 = 0xFF51AFD7ED558CCD
_C2 = 0xC4CEB9FE1A85EC53
_MASK64 = (1 << 64) - 1


def block_classes(w: Workload) -> np.ndarray:
    """Drawn class of each (h, qb, kb) block of the mask: 0 empty, 1 partial, 2 full, with
    probabilities (p_empty, p_partial, p_full)."""
    rng = rng_for(w.seed + 2000)
    nqb, nkb = -(-w.q_len // w.block), -(-w.kv_len // w.block)
    u = rng.random(size=(w.nheads, nqb, nkb))
    cls = np.full(u.shape, 1, dtype=np.uint8)
    cls[u < w.p_empty] = 0
    cls[u >= w.p_empty + w.p_partial] = 2
    return cls


def _fmix64_np(k: np.ndarray) -> np.ndarray:
    k = k.astype(np.uint64)
    k ^= k >> np.uint64(33)
    k *= np.uint64(_C1)
    k ^= k >> np.uint64(33)
    k *= np.uint64(_C2)
    k ^= k >> np.uint64(33)
    return k


def _signed(c: int) -> int:
    return c - (1 << 64) if c >= (1 << 63) else c


def _fmix64_torch(k: torch.Tensor) -> torch.Tensor:
    """fmix64 on int64 tensors (two's-complement wrap-around; logical shifts emulated)."""
    lo31 = (1 << 31) - 1  # a logical right shift by 33 keeps 31 bits
    k = k ^ ((k >> 33) & lo31)
    k = k * _signed(_C1)
    k = k ^ ((k >> 33) & lo31)
    k = k * _signed(_C2)
    k = k ^ ((k >> 33) & lo31)
    return k


def mask_rows(w: Workload, cls: np.ndarray, h: int, rows) -> np.ndarray:
    """Rows `rows` of head h of the mask, uint8 (len(rows), Lk), on the host.
    Bit (h, i, j) of a partial block is the top bit of fmix64(((seed*H + h)*Lq + i)*Lk + j);
    the diagonal i == j is then set to 1 (every row keeps a key)."""
    rows = np.asarray(rows, dtype=np.int64)
    j = np.arange(w.kv_len, dtype=np.int64)
    kb = j // w.block
    out = np.empty((len(rows), w.kv_len), dtype=np.uint8)
    for r, i in enumerate(rows):
        c = cls[h, i // w.block, kb]
        key = ((np.uint64(w.seed) * np.uint64(w.nheads) + np.uint64(h)) * np.uint64(w.q_len)
               + np.uint64(i)) * np.uint64(w.kv_len) + j.astype(np.uint64)
        bit = (_fmix64_np(key) >> np.uint64(63)).astype(np.uint8)
        row = np.where(c == 2, 1, np.where(c == 0, 0, bit)).astype(np.uint8)
        if i < w.kv_len:
            row[i] = 1
        out[r] = row
    return out


def mask_device(w: Workload, cls: np.ndarray, device) -> torch.Tensor:
    """The whole mask (H, Lq, Lk) uint8 built on `device` with torch, head by head and in
    row chunks; identical to mask_rows() element by element."""
    H, Lq, Lk, blk = w.nheads, w.q_len, w.kv_len, w.block
    out = torch.empty((H, Lq, Lk), dtype=torch.uint8, device=device)
    cls_t = torch.from_numpy(cls.astype(np.int64)).to(device)
    j = torch.arange(Lk, dtype=torch.int64, device=device)
    chunk = max(1, (1 << 26) // max(Lk, 1))
    for h in range(H):
        for i0 in range(0, Lq, chunk):
            i = torch.arange(i0, min(Lq, i0 + chunk), dtype=torch.int64, device=device)
            key = ((w.seed * H + h) * Lq + i[:, None]) * Lk + j[None, :]
            bit = (_fmix64_torch(key) < 0).to(torch.uint8)
            c = cls_t[h][(i // blk)[:, None], (j // blk)[None, :]]
            row = torch.where(c == 2, torch.ones_like(bit), torch.where(c == 0, torch.zeros_like(bit), bit))
            diag = (i[:, None] == j[None, :])
            row = torch.where(diag, torch.ones_like(row), row)
            out[h, i0:i0 + len(i)] = row
    return out


def packed_segments(w: Workload) -> list:
    """Sequence lengths, uniform in [seg_min, seg_max], adding up to w.q_len (the last one is
    cut to fit)."""
    rng = rng_for(w.seed + 1)
    segs, total = [], 0
    while total < w.q_len:
        n = int(min(rng.integers(w.seg_min, w.seg_max + 1), w.q_len - total))
        segs.append(n)
        total += n
    return segs


def packed_qkv(w: Workload):
    """q (total, nheads, head_dim), k and v (total, nkvheads, head_dim), i.i.d. N(0, 1)."""
    rng = rng_for(w.seed)
    return (normal(rng, (w.q_len, w.nheads, w.head_dim), w.dtype),
            normal(rng, (w.kv_len, w.nkvheads, w.head_dim), w.dtype),
            normal(rng, (w.kv_len, w.nkvheads, w.head_dim), w.dtype))
