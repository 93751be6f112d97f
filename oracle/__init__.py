"""CPU float64 oracle for scaled-dot-product attention — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package. The CUDA library and its Python binding never import it, and the two
share no code.

The arithmetic lives in ``sdpa_oracle.c`` (plain loops, float64, two-pass softmax); this
module compiles it with gcc and marshals numpy arrays into it. Arrays use the row-major
layout (batch, seq_len, nheads, head_dim), which is the same memory as the column-major
(head_dim, nheads, seq_len, batch) of the Flux.jl page "Neural Network primitives from
NNlib.jl" (scaled_dot_product_attention, first paragraphs).

Parity of every function is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sdpa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_sdpa.so")
_lock = threading.Lock()
_lib = None

_i64p = ctypes.POINTER(ctypes.c_int64)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_i32p = ctypes.POINTER(ctypes.c_int32)


class _Problem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64), ("q_len", ctypes.c_int64), ("kv_len", ctypes.c_int64),
        ("nheads", ctypes.c_int64), ("nkvheads", ctypes.c_int64), ("dqk", ctypes.c_int64),
        ("dv", ctypes.c_int64), ("scale", ctypes.c_double), ("causal", ctypes.c_int32),
        ("kv_head_rule", ctypes.c_int32), ("q_offset_scalar", ctypes.c_int64),
        ("q_offset", _i64p), ("q_lengths", _i64p), ("kv_lengths", _i64p),
        ("bias", _f64p), ("bias_stride", ctypes.c_int64 * 4),
        ("mask", _u8p), ("mask_stride", ctypes.c_int64 * 4),
    ]


def build(source: str = _SRC, output: str = _LIB, force: bool = False,
          extra_flags: tuple = ()) -> str:
    """Compile the C oracle into a shared library (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(output) or os.path.getmtime(output) < os.path.getmtime(source):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", *extra_flags,
               "-o", output, source, "-lm"]
        subprocess.run(cmd, check=True)
    return output


def load(path: str | None = None):
    """Load (building if needed) the oracle library and declare its signatures."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    with _lock:
        lib_path = path or build()
        lib = ctypes.CDLL(lib_path)
        lib.oracle_sdpa_forward.argtypes = [ctypes.POINTER(_Problem), _f64p, _f64p, _f64p, _f64p]
        lib.oracle_sdpa_forward.restype = ctypes.c_int
        lib.oracle_sdpa_forward_lse.argtypes = [ctypes.POINTER(_Problem), _f64p, _f64p, _f64p, _f64p, _f64p]
        lib.oracle_sdpa_forward_lse.restype = ctypes.c_int
        lib.oracle_rope.argtypes = [_f64p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, _i64p,
                                    ctypes.c_double, _f64p]
        lib.oracle_rope.restype = ctypes.c_int
        lib.oracle_sdpa_forward_with_weights.argtypes = [
            ctypes.POINTER(_Problem), _f64p, _f64p, _f64p, ctypes.c_double, ctypes.c_uint64, _f64p, _f64p]
        lib.oracle_sdpa_forward_with_weights.restype = ctypes.c_int
        lib.oracle_sdpa_backward.argtypes = [
            ctypes.POINTER(_Problem), _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p]
        lib.oracle_sdpa_backward.restype = ctypes.c_int
        lib.oracle_sdpa_forward_packed.argtypes = [
            ctypes.POINTER(_Problem), ctypes.c_int64, _i64p, _i64p, ctypes.c_int64, _f64p, _f64p,
            _f64p, _f64p]
        lib.oracle_sdpa_forward_packed.restype = ctypes.c_int
        lib.oracle_cache_update_at_index.argtypes = [
            _f64p, _f64p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_int64, _i64p]
        lib.oracle_cache_update_at_index.restype = ctypes.c_int
        lib.oracle_sdpa_decode_with_cache.argtypes = [
            ctypes.POINTER(_Problem), _f64p, _f64p, _f64p, _f64p, _f64p, _i64p, _f64p]
        lib.oracle_sdpa_decode_with_cache.restype = ctypes.c_int
        lib.oracle_block_mask_info.argtypes = [
            _u8p, _i64p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_int64, _u8p, _i32p, _u32p, _u32p]
        lib.oracle_block_mask_info.restype = ctypes.c_int
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ctypes.c_int
        if path is None:
            _lib = lib
        return lib


class OracleError(RuntimeError):
    pass


def max_threads() -> int:
    return int(load().oracle_max_threads())


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _per_batch(x, batch: int):
    """An integer or per-batch integer array -> int64 array of `batch` entries, or None."""
    if x is None:
        return None
    arr = np.asarray(x, dtype=np.int64)
    if arr.ndim == 0:
        arr = np.full((batch,), int(arr), dtype=np.int64)
    if arr.shape != (batch,):
        raise ValueError(f"expected {batch} per-batch entries, got shape {arr.shape}")
    return np.ascontiguousarray(arr)


def _broadcast4(a, dtype, batch, nheads, q_len, kv_len):
    """Broadcast `a` to row-major (batch, nheads, q_len, kv_len), which is the page's
    column-major (kv_len, q_len, nheads, batch). Returns the base array and its element
    strides in the order (key j, query i, head h, batch b)."""
    base = np.ascontiguousarray(np.asarray(a, dtype=dtype))
    while base.ndim < 4:
        base = base[None]
    view = np.broadcast_to(base, (batch, nheads, q_len, kv_len))
    es = base.itemsize
    sb, sh, si, sj = (s // es for s in view.strides)
    return base, (sj, si, sh, sb)


def sdpa_forward_lse(q, k, v, bias=None, mask=None, scale=None, is_causal=False, q_offset=0,
                     q_lengths=None, kv_lengths=None, kv_head_rule: str = "contiguous", lib=None):
    """sdpa_forward, and each row's log-sum-exp (natural log of the softmax's normaliser over the
    attended keys; +inf for a row with no key or past q_lengths) as (B, H, Lq)."""
    return sdpa_forward(q, k, v, bias, mask, scale, is_causal, q_offset, q_lengths, kv_lengths, kv_head_rule,
                        lib, _with_lse=True)


def sdpa_forward(q, k, v, bias=None, mask=None, scale=None, is_causal=False, q_offset=0,
                 q_lengths=None, kv_lengths=None, kv_head_rule: str = "contiguous",
                 lib=None, _with_lse=False) -> np.ndarray:
    """scaled_dot_product_attention(query, key, value, [bias]; mask, scale, is_causal,
    q_offset, q_lengths, kv_lengths) in float64.

    q: (B, Lq, H, dqk); k: (B, Lk, Hkv, dqk); v: (B, Lk, Hkv, dv); returns (B, Lq, H, dv).
    bias / mask: broadcastable to row-major (B, H, Lq, Lk). is_causal: False, True or
    "bottom_right". kv_head_rule: "contiguous" (h // (H/Hkv)) or "interleaved" (h % Hkv).
    """
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Lq, H, D = q.shape
    Bk, Lk, Hkv, Dk = k.shape
    Dv = v.shape[3]
    if Bk != B or v.shape[:3] != (B, Lk, Hkv) or Dk != D:
        raise ValueError("inconsistent q/k/v shapes")
    p = _Problem()
    p.batch, p.q_len, p.kv_len, p.nheads, p.nkvheads, p.dqk, p.dv = B, Lq, Lk, H, Hkv, D, Dv
    p.scale = float("nan") if scale is None else float(scale)
    p.causal = {False: 0, True: 1, "bottom_right": 2}[is_causal]
    p.kv_head_rule = {"contiguous": 0, "interleaved": 1}[kv_head_rule]
    keep = []
    qo = np.asarray(q_offset, dtype=np.int64)
    if qo.ndim == 0:
        p.q_offset_scalar = int(qo)
    else:
        qo = _per_batch(qo, B)
        keep.append(qo)
        p.q_offset = _ptr(qo, _i64p)
    for name, val in (("q_lengths", q_lengths), ("kv_lengths", kv_lengths)):
        arr = _per_batch(val, B)
        if arr is not None:
            keep.append(arr)
            setattr(p, name, _ptr(arr, _i64p))
    if bias is not None:
        base, st = _broadcast4(bias, np.float64, B, H, Lq, Lk)
        keep.append(base)
        p.bias = _ptr(base, _f64p)
        p.bias_stride = (ctypes.c_int64 * 4)(*st)
    if mask is not None:
        base, st = _broadcast4(np.asarray(mask).astype(np.uint8), np.uint8, B, H, Lq, Lk)
        keep.append(base)
        p.mask = _ptr(base, _u8p)
        p.mask_stride = (ctypes.c_int64 * 4)(*st)
    out = np.empty((B, Lq, H, Dv), dtype=np.float64)
    if _with_lse:
        lse = np.empty((B, H, Lq), dtype=np.float64)
        rc = lib.oracle_sdpa_forward_lse(ctypes.byref(p), _ptr(q, _f64p), _ptr(k, _f64p),
                                         _ptr(v, _f64p), _ptr(out, _f64p), _ptr(lse, _f64p))
        if rc != 0:
            raise OracleError(f"oracle_sdpa_forward_lse failed with code {rc}")
        return out, lse
    rc = lib.oracle_sdpa_forward(ctypes.byref(p), _ptr(q, _f64p), _ptr(k, _f64p),
                                 _ptr(v, _f64p), _ptr(out, _f64p))
    if rc != 0:
        raise OracleError(f"oracle_sdpa_forward failed with code {rc}")
    return out


def rope(x, positions, base=10000.0, lib=None) -> np.ndarray:
    """Rotary position embedding of x (..., nheads, d), positions one per row of the leading
    dimensions: the pair (c, c + d/2) rotated by positions[t] * base^(-2c/d)."""
    lib = lib or load()
    x = _f64(x)
    *lead, H, d = x.shape
    rows = int(np.prod(lead)) if lead else 1
    pos = np.ascontiguousarray(np.asarray(positions, dtype=np.int64).reshape(-1))
    if pos.shape != (rows,):
        raise ValueError(f"expected {rows} positions, got {pos.shape}")
    out = np.empty_like(x)
    rc = lib.oracle_rope(_ptr(x, _f64p), rows, H, d, _ptr(pos, _i64p), float(base), _ptr(out, _f64p))
    if rc != 0:
        raise OracleError(f"oracle_rope failed with code {rc}")
    return out


def sdpa_forward_with_weights(q, k, v, bias=None, mask=None, scale=None, is_causal=False, q_offset=0,
                              q_lengths=None, kv_lengths=None, drop_p=0.0, seed=0, lib=None):
    """scaled_dot_product_attention_with_weights(query, key, value, [bias]; fdrop, mask, scale,
    is_causal, q_offset, q_lengths, kv_lengths) in float64, with fdrop = dropout of probability
    drop_p drawn by the counter-based generator of the C source (seeded by `seed`). Returns
    (out (B, Lq, H, dv), weights (B, H, Lq, Lk)): the weights after the dropout, the page's
    (kv_len, q_len, nheads, batch) order."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Lq, H, D = q.shape
    Bk, Lk, Hkv, Dk = k.shape
    Dv = v.shape[3]
    if Bk != B or v.shape[:3] != (B, Lk, Hkv) or Dk != D:
        raise ValueError("inconsistent q/k/v shapes")
    p = _Problem()
    p.batch, p.q_len, p.kv_len, p.nheads, p.nkvheads, p.dqk, p.dv = B, Lq, Lk, H, Hkv, D, Dv
    p.scale = float("nan") if scale is None else float(scale)
    p.causal = {False: 0, True: 1, "bottom_right": 2}[is_causal]
    keep = []
    qo = np.asarray(q_offset, dtype=np.int64)
    if qo.ndim == 0:
        p.q_offset_scalar = int(qo)
    else:
        qo = _per_batch(qo, B)
        keep.append(qo)
        p.q_offset = _ptr(qo, _i64p)
    for name, val in (("q_lengths", q_lengths), ("kv_lengths", kv_lengths)):
        arr = _per_batch(val, B)
        if arr is not None:
            keep.append(arr)
            setattr(p, name, _ptr(arr, _i64p))
    if bias is not None:
        base, st = _broadcast4(bias, np.float64, B, H, Lq, Lk)
        keep.append(base)
        p.bias = _ptr(base, _f64p)
        p.bias_stride = (ctypes.c_int64 * 4)(*st)
    if mask is not None:
        base, st = _broadcast4(np.asarray(mask).astype(np.uint8), np.uint8, B, H, Lq, Lk)
        keep.append(base)
        p.mask = _ptr(base, _u8p)
        p.mask_stride = (ctypes.c_int64 * 4)(*st)
    out = np.empty((B, Lq, H, Dv), dtype=np.float64)
    weights = np.empty((B, H, Lq, Lk), dtype=np.float64)
    rc = lib.oracle_sdpa_forward_with_weights(ctypes.byref(p), _ptr(q, _f64p), _ptr(k, _f64p),
                                              _ptr(v, _f64p), float(drop_p), int(seed) & (2**64 - 1),
                                              _ptr(out, _f64p), _ptr(weights, _f64p))
    if rc != 0:
        raise OracleError(f"oracle_sdpa_forward_with_weights failed with code {rc}")
    return out, weights


def sdpa_backward(q, k, v, dout, mask=None, scale=None, is_causal=False, q_offset=0,
                  q_lengths=None, kv_lengths=None, lib=None):
    """Gradient of the fused implementation for the loss sum(dout * out): returns
    (dq, dk, dv, dscale) in float64, with the shapes of q, k, v and a float. Rows with no
    attended key and rows past q_lengths take no part. No bias (a call with a bias takes the
    materialized implementation under automatic differentiation)."""
    lib = lib or load()
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Lq, H, D = q.shape
    Bk, Lk, Hkv, Dk = k.shape
    Dv = v.shape[3]
    if Bk != B or v.shape[:3] != (B, Lk, Hkv) or Dk != D or dout.shape != (B, Lq, H, Dv):
        raise ValueError("inconsistent q/k/v/dout shapes")
    p = _Problem()
    p.batch, p.q_len, p.kv_len, p.nheads, p.nkvheads, p.dqk, p.dv = B, Lq, Lk, H, Hkv, D, Dv
    p.scale = float("nan") if scale is None else float(scale)
    p.causal = {False: 0, True: 1, "bottom_right": 2}[is_causal]
    keep = []
    qo = np.asarray(q_offset, dtype=np.int64)
    if qo.ndim == 0:
        p.q_offset_scalar = int(qo)
    else:
        qo = _per_batch(qo, B)
        keep.append(qo)
        p.q_offset = _ptr(qo, _i64p)
    for name, val in (("q_lengths", q_lengths), ("kv_lengths", kv_lengths)):
        arr = _per_batch(val, B)
        if arr is not None:
            keep.append(arr)
            setattr(p, name, _ptr(arr, _i64p))
    if mask is not None:
        base, st = _broadcast4(np.asarray(mask).astype(np.uint8), np.uint8, B, H, Lq, Lk)
        keep.append(base)
        p.mask = _ptr(base, _u8p)
        p.mask_stride = (ctypes.c_int64 * 4)(*st)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    ds = np.zeros(1, dtype=np.float64)
    rc = lib.oracle_sdpa_backward(ctypes.byref(p), _ptr(q, _f64p), _ptr(k, _f64p), _ptr(v, _f64p),
                                  _ptr(dout, _f64p), _ptr(dq, _f64p), _ptr(dk, _f64p), _ptr(dv, _f64p),
                                  _ptr(ds, _f64p))
    if rc != 0:
        raise OracleError(f"oracle_sdpa_backward failed with code {rc}")
    return dq, dk, dv, float(ds[0])


def sdpa_forward_packed(q, k, v, q_segments, kv_segments=None, maxlen=None, scale=None,
                        is_causal=False, q_offset=0, q_lengths=None, kv_lengths=None,
                        kv_head_rule: str = "contiguous", lib=None) -> np.ndarray:
    """scaled_dot_product_attention(query, key, value; q_segments, kv_segments, maxlen, scale,
    is_causal, q_offset, q_lengths, kv_lengths) on packed sequences, in float64.

    q: (total_q, H, dqk); k: (total_kv, Hkv, dqk); v: (total_kv, Hkv, dv), the sequences one
    after the other with no batch axis; returns (total_q, H, dv). q_segments / kv_segments:
    the lengths of the sequences (kv_segments defaults to q_segments); q_offset, q_lengths
    and kv_lengths take one entry per sequence (or one integer for all).
    """
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    Lq, H, D = q.shape
    Lk, Hkv, Dk = k.shape
    Dv = v.shape[2]
    if v.shape[:2] != (Lk, Hkv) or Dk != D:
        raise ValueError("inconsistent q/k/v shapes")
    qs = np.ascontiguousarray(np.asarray(q_segments, dtype=np.int64).reshape(-1))
    nseg = qs.shape[0]
    ks = None if kv_segments is None else np.ascontiguousarray(
        np.asarray(kv_segments, dtype=np.int64).reshape(-1))
    if ks is not None and ks.shape != (nseg,):
        raise ValueError("kv_segments must have one entry per query segment")
    p = _Problem()
    p.batch, p.q_len, p.kv_len, p.nheads, p.nkvheads, p.dqk, p.dv = 1, Lq, Lk, H, Hkv, D, Dv
    p.scale = float("nan") if scale is None else float(scale)
    p.causal = {False: 0, True: 1, "bottom_right": 2}[is_causal]
    p.kv_head_rule = {"contiguous": 0, "interleaved": 1}[kv_head_rule]
    keep = [qs] + ([ks] if ks is not None else [])
    qo = np.asarray(q_offset, dtype=np.int64)
    if qo.ndim == 0:
        p.q_offset_scalar = int(qo)
    else:
        qo = _per_batch(qo, nseg)
        keep.append(qo)
        p.q_offset = _ptr(qo, _i64p)
    for name, val in (("q_lengths", q_lengths), ("kv_lengths", kv_lengths)):
        arr = _per_batch(val, nseg)
        if arr is not None:
            keep.append(arr)
            setattr(p, name, _ptr(arr, _i64p))
    out = np.zeros((Lq, H, Dv), dtype=np.float64)
    rc = lib.oracle_sdpa_forward_packed(
        ctypes.byref(p), nseg, _ptr(qs, _i64p), None if ks is None else _ptr(ks, _i64p),
        -1 if maxlen is None else int(maxlen), _ptr(q, _f64p), _ptr(k, _f64p), _ptr(v, _f64p),
        _ptr(out, _f64p))
    if rc != 0:
        raise OracleError(f"oracle_sdpa_forward_packed failed with code {rc}")
    return out


def cache_update_at_index(cache, new_rows, index, lib=None) -> np.ndarray:
    """Returns a copy of `cache` (B, capacity, Hkv, d) with new_rows (B, n_new, Hkv, d)
    written at positions index[b] .. index[b] + n_new - 1."""
    lib = lib or load()
    cache = _f64(cache).copy()
    new_rows = _f64(new_rows)
    B, cap, Hkv, d = cache.shape
    n_new = new_rows.shape[1]
    if new_rows.shape != (B, n_new, Hkv, d):
        raise ValueError("new rows do not match the cache")
    idx = _per_batch(index, B)
    rc = lib.oracle_cache_update_at_index(_ptr(cache, _f64p), _ptr(new_rows, _f64p), B, cap,
                                          n_new, Hkv, d, _ptr(idx, _i64p))
    if rc != 0:
        raise OracleError(f"oracle_cache_update_at_index failed with code {rc}")
    return cache


def sdpa_decode_with_cache(q, k_new, v_new, k_cache, v_cache, index, scale=None,
                           lib=None):
    """Write k_new/v_new into copies of the caches at `index`, then attend with
    :bottom_right causal alignment over kv_lengths = index + n_new.
    Returns (out, k_cache_after, v_cache_after)."""
    lib = lib or load()
    q = _f64(q)
    k_new, v_new = _f64(k_new), _f64(v_new)
    kc, vc = _f64(k_cache).copy(), _f64(v_cache).copy()
    B, n_new, H, D = q.shape
    _, cap, Hkv, _ = kc.shape
    Dv = vc.shape[3]
    idx = _per_batch(index, B)
    p = _Problem()
    p.batch, p.q_len, p.kv_len, p.nheads, p.nkvheads, p.dqk, p.dv = B, n_new, cap, H, Hkv, D, Dv
    p.scale = float("nan") if scale is None else float(scale)
    p.causal = 2
    p.kv_head_rule = 0
    out = np.empty((B, n_new, H, Dv), dtype=np.float64)
    rc = lib.oracle_sdpa_decode_with_cache(
        ctypes.byref(p), _ptr(q, _f64p), _ptr(k_new, _f64p), _ptr(v_new, _f64p),
        _ptr(kc, _f64p), _ptr(vc, _f64p), _ptr(idx, _i64p), _ptr(out, _f64p))
    if rc != 0:
        raise OracleError(f"oracle_sdpa_decode_with_cache failed with code {rc}")
    return out, kc, vc


def block_mask_info(mask, bq: int = 128, bk: int = 128, lib=None) -> dict:
    """Classify the blocks of a boolean mask of row-major shape (H, Lq, Lk).

    Returns dict(cls=(H, nqb, nkb) uint8 [0 empty, 1 partial, 2 full],
    count=(H, nqb) int32, list=(H, nqb, nkb) uint32 [kb | cls << 30 for the first count
    entries], bits=(H, nqb, nkb, bq, ceil(bk/32)) uint32 [meaningful for partial blocks]).
    """
    lib = lib or load()
    m = np.ascontiguousarray(np.asarray(mask).astype(np.uint8))
    H, Lq, Lk = m.shape
    nqb, nkb, words = -(-Lq // bq), -(-Lk // bk), -(-bk // 32)
    ms = np.array([1, Lk, Lq * Lk], dtype=np.int64)
    cls = np.zeros((H, nqb, nkb), dtype=np.uint8)
    count = np.zeros((H, nqb), dtype=np.int32)
    lst = np.zeros((H, nqb, nkb), dtype=np.uint32)
    bits = np.zeros((H, nqb, nkb, bq, words), dtype=np.uint32)
    rc = lib.oracle_block_mask_info(_ptr(m, _u8p), _ptr(ms, _i64p), H, Lq, Lk, bq, bk,
                                    _ptr(cls, _u8p), _ptr(count, _i32p), _ptr(lst, _u32p),
                                    _ptr(bits, _u32p))
    if rc != 0:
        raise OracleError(f"oracle_block_mask_info failed with code {rc}")
    return dict(cls=cls, count=count, list=lst, bits=bits)
