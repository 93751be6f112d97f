"""Python binding of libsdpa.so: multi-head scaled-dot-product attention on B200 (sm_100a).

Argument marshalling only: torch tensors provide device memory and the current stream; every
step of the computation runs in the library's CUDA kernels. The functions mirror the C ABI in
include/sdpa.h (same names), which restates NNlib.scaled_dot_product_attention from the Flux.jl
page "Neural Network primitives from NNlib.jl".

Layout: q (B, Lq, H, dqk), k (B, Lk, Hkv, dqk), v (B, Lk, Hkv, dv), out (B, Lq, H, dv) —
row-major, i.e. the page's column-major (head_dim, nheads, seq_len, batch). A bias or mask is
broadcastable to row-major (B, H, Lq, Lk), the page's (kv_len, q_len, nheads, batch).

There is no fallback: if libsdpa.so is missing, importing this package raises. With
SDPA_DEBUG_CHECKS=1 in the environment the package loads libsdpa_debug.so instead: the same
kernels with every data-dependent device index range-checked (a violation is recorded as
SDPA_ERR_DEVICE_CHECK in the status word instead of an out-of-range access).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
DEBUG_CHECKS = os.environ.get("SDPA_DEBUG_CHECKS", "0") not in ("", "0")
LIB_PATH = os.path.join(_HERE, "libsdpa_debug.so" if DEBUG_CHECKS else "libsdpa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing; build it with `python head_scaled_dot_sdpa_b200/build.py"
        f"{' --debug-checks' if DEBUG_CHECKS else ''}`")
_lib = ctypes.CDLL(LIB_PATH)

# ---- ABI mirror -------------------------------------------------------------------------------

SDPA_OK, SDPA_ERR_INVALID_ARG, SDPA_ERR_UNSUPPORTED, SDPA_ERR_WORKSPACE = 0, 1, 2, 3
SDPA_ERR_CUDA, SDPA_ERR_TIMEOUT, SDPA_ERR_DEVICE_CHECK = 4, 5, 6
STATUS_NAMES = {0: "SDPA_OK", 1: "SDPA_ERR_INVALID_ARG", 2: "SDPA_ERR_UNSUPPORTED",
                3: "SDPA_ERR_WORKSPACE", 4: "SDPA_ERR_CUDA", 5: "SDPA_ERR_TIMEOUT",
                6: "SDPA_ERR_DEVICE_CHECK"}
SDPA_F32, SDPA_F16, SDPA_BF16 = 0, 1, 2
SDPA_CAUSAL_NONE, SDPA_CAUSAL_TOP_LEFT, SDPA_CAUSAL_BOTTOM_RIGHT = 0, 1, 2
SDPA_FLAG_GENERIC_KERNEL = 0x1
SDPA_FLAG_SELFTEST_STALL = 0x2
SDPA_BLOCK_EMPTY, SDPA_BLOCK_PARTIAL, SDPA_BLOCK_FULL = 0, 1, 2

_DTYPE = {torch.float32: SDPA_F32, torch.float16: SDPA_F16, torch.bfloat16: SDPA_BF16}


class BlockMaskInfoStruct(ctypes.Structure):
    _fields_ = [("nheads", ctypes.c_int32), ("q_len", ctypes.c_int32), ("kv_len", ctypes.c_int32),
                ("bq", ctypes.c_int32), ("bk", ctypes.c_int32), ("nqb", ctypes.c_int32),
                ("nkb", ctypes.c_int32), ("block_class", ctypes.c_void_p),
                ("row_count", ctypes.c_void_p), ("row_list", ctypes.c_void_p),
                ("partial_bits", ctypes.c_void_p)]


class Params(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("batch", ctypes.c_int32), ("q_len", ctypes.c_int32),
                ("kv_len", ctypes.c_int32), ("nheads", ctypes.c_int32),
                ("nkvheads", ctypes.c_int32), ("dqk", ctypes.c_int32), ("dv", ctypes.c_int32),
                ("scale", ctypes.c_float), ("causal", ctypes.c_int),
                ("q_offset_scalar", ctypes.c_int32), ("q_offset", ctypes.c_void_p),
                ("q_lengths", ctypes.c_void_p), ("kv_lengths", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("bias_dtype", ctypes.c_int),
                ("bias_stride", ctypes.c_int64 * 4), ("mask", ctypes.c_void_p),
                ("mask_stride", ctypes.c_int64 * 4),
                ("block_info", ctypes.POINTER(BlockMaskInfoStruct)), ("flags", ctypes.c_uint32)]


class PackedSegments(ctypes.Structure):
    _fields_ = [("nseg", ctypes.c_int32), ("maxlen", ctypes.c_int32), ("q_segments", ctypes.c_void_p),
                ("kv_segments", ctypes.c_void_p)]


_vp, _sz, _i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
_PP = ctypes.POINTER(Params)
_lib.sdpa_workspace_size.argtypes = [_PP]
_lib.sdpa_workspace_size.restype = _sz
_lib.sdpa_workspace_init.argtypes = [_vp, _sz, _vp]
_lib.sdpa_forward.argtypes = [_PP, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sdpa_packed_workspace_size.argtypes = [_PP, ctypes.POINTER(PackedSegments)]
_lib.sdpa_packed_workspace_size.restype = _sz
_lib.sdpa_forward_packed.argtypes = [_PP, ctypes.POINTER(PackedSegments), _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sdpa_forward_with_weights.argtypes = [_PP, ctypes.c_double, ctypes.c_uint64, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                           _vp]
_lib.sdpa_rope.argtypes = [_vp, _vp, ctypes.c_int, ctypes.c_int64, _i32, _i32, _vp, ctypes.c_double, _vp]
_lib.sdpa_backward_workspace_size.argtypes = [_PP]
_lib.sdpa_backward_workspace_size.restype = _sz
_lib.sdpa_weights_workspace_size.argtypes = [_PP]
_lib.sdpa_weights_workspace_size.restype = _sz
_lib.sdpa_rope_workspace_size.argtypes = [_PP]
_lib.sdpa_rope_workspace_size.restype = _sz
_lib.sdpa_forward_rope.argtypes = [_PP, _vp, _vp, ctypes.c_double, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sdpa_backward.argtypes = [_PP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sdpa_backward_lse.argtypes = [_PP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sdpa_forward_lse.argtypes = [_PP, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sdpa_decode_with_cache.argtypes = [_PP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.cache_update_at_index.argtypes = [_vp, _vp, _vp, _vp, ctypes.c_int, _i32, _i32, _i32, _i32,
                                       _i32, _vp, _vp, _vp]
_lib.build_block_mask_info_size.argtypes = [_i32] * 5
_lib.build_block_mask_info_size.restype = _sz
_lib.build_block_mask_info.argtypes = [_vp, ctypes.POINTER(ctypes.c_int64), _i32, _i32, _i32, _i32,
                                       _i32, _vp, _sz, ctypes.POINTER(BlockMaskInfoStruct), _vp]
_lib.sdpa_read_device_status.argtypes = [_vp, _vp]
_lib.sdpa_last_error.restype = ctypes.c_char_p
_lib.sdpa_last_kernel.restype = ctypes.c_char_p
for _f in ("sdpa_workspace_init", "sdpa_forward", "sdpa_forward_packed", "sdpa_forward_with_weights",
           "sdpa_rope", "sdpa_backward", "sdpa_decode_with_cache",
           "cache_update_at_index",
           "build_block_mask_info", "sdpa_read_device_status"):
    getattr(_lib, _f).restype = ctypes.c_int

lib = _lib  # the raw ctypes handle (tests call the C ABI through it)


class SdpaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def _check(status: int):
    if status != SDPA_OK:
        raise SdpaError(status, _lib.sdpa_last_error().decode())


def last_kernel() -> str:
    return _lib.sdpa_last_kernel().decode()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


# ---- workspace ----------------------------------------------------------------------------------

class Workspace:
    """Caller-owned scratch (device status word + kernel scratch), grown on demand. The status
    word starts at SDPA_OK; read_device_status() returns and clears it."""

    def __init__(self, device=None, nbytes: int = 1 << 20):
        self.device = torch.device(device or "cuda")
        self.buf = None
        self._grow(nbytes)

    def _grow(self, nbytes: int):
        nbytes = max(256, (nbytes + 255) // 256 * 256)
        self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=self.device)
        off = (-self.buf.data_ptr()) % 256
        self.view = self.buf[off:off + nbytes]
        # a new buffer starts with a clear status word
        _check(_lib.sdpa_workspace_init(self.ptr, self.nbytes, _stream(None)))

    @property
    def ptr(self) -> int:
        return self.view.data_ptr()

    @property
    def nbytes(self) -> int:
        return self.view.numel()

    def ensure(self, nbytes: int):
        if nbytes > self.nbytes:
            self._grow(nbytes)
        return self


_default_ws = {}


def _workspace(device, need: int, ws: Workspace | None) -> Workspace:
    if ws is None:
        key = torch.device(device).index or 0
        ws = _default_ws.get(key)
        if ws is None:
            ws = _default_ws[key] = Workspace(device, max(need, 1 << 20))
    return ws.ensure(need)


def read_device_status(ws: Workspace | None = None, stream=None) -> int:
    """Synchronises and returns (then clears) the device status word of the workspace."""
    ws = ws or _default_ws.get(torch.cuda.current_device())
    if ws is None:
        return SDPA_OK
    return int(_lib.sdpa_read_device_status(ws.ptr, _stream(stream)))


# ---- argument marshalling -----------------------------------------------------------------------

def _per_batch(x, batch: int, device, name: str):
    """An int -> scalar; a sequence or tensor -> device int32 [batch]."""
    if x is None:
        return None
    if isinstance(x, int):
        return torch.full((batch,), x, dtype=torch.int32, device=device)
    t = torch.as_tensor(x, dtype=torch.int32, device=device)
    if t.shape != (batch,):
        raise ValueError(f"{name} must have {batch} entries, got {tuple(t.shape)}")
    return t.contiguous()


def _broadcast_strides(t: torch.Tensor, B, H, Lq, Lk):
    """Element strides (j, i, h, b) of `t` broadcast to row-major (B, H, Lq, Lk)."""
    while t.dim() < 4:
        t = t.unsqueeze(0)
    e = t.expand(B, H, Lq, Lk)
    sb, sh, si, sj = e.stride()
    return (sj, si, sh, sb)


def _params(q, k, v, *, bias, mask, scale, is_causal, q_offset, q_lengths, kv_lengths, block_info,
            flags, keep):
    B, Lq, H, D = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    p = Params()
    p.dtype = _DTYPE[q.dtype]
    p.batch, p.q_len, p.kv_len, p.nheads, p.nkvheads, p.dqk, p.dv = B, Lq, Lk, H, Hkv, D, v.shape[3]
    p.scale = float("nan") if scale is None else float(scale)
    p.causal = {False: SDPA_CAUSAL_NONE, True: SDPA_CAUSAL_TOP_LEFT,
                "bottom_right": SDPA_CAUSAL_BOTTOM_RIGHT}[is_causal]
    dev = q.device
    if isinstance(q_offset, int):
        p.q_offset_scalar = q_offset
    else:
        t = _per_batch(q_offset, B, dev, "q_offset")
        keep.append(t)
        p.q_offset = t.data_ptr()
    for name, val in (("q_lengths", q_lengths), ("kv_lengths", kv_lengths)):
        t = _per_batch(val, B, dev, name)
        if t is not None:
            keep.append(t)
            setattr(p, name, t.data_ptr())
    if bias is not None:
        if bias.dtype not in _DTYPE or bias.device != dev:
            raise ValueError("bias must be a float tensor on the device of q")
        p.bias = bias.data_ptr()
        p.bias_dtype = _DTYPE[bias.dtype]
        p.bias_stride = (ctypes.c_int64 * 4)(*_broadcast_strides(bias, B, H, Lq, Lk))
    if mask is not None:
        if mask.dtype not in (torch.bool, torch.uint8) or mask.device != dev:
            raise ValueError("mask must be a bool/uint8 tensor on the device of q")
        p.mask = mask.data_ptr()
        p.mask_stride = (ctypes.c_int64 * 4)(*_broadcast_strides(mask, B, H, Lq, Lk))
    if block_info is not None:
        p.block_info = ctypes.pointer(block_info.struct)
        keep.append(block_info)
    p.flags = flags
    return p


def _check_qkv(q, k, v):
    for n, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{n} must be a contiguous 4-d CUDA tensor (B, L, H, d)")
        if t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, k and v must share dtype and device")
    if k.shape[0] != q.shape[0] or v.shape[:3] != k.shape[:3] or k.shape[3] != q.shape[3]:
        raise ValueError("inconsistent q/k/v shapes")


def sdpa_forward(q, k, v, bias=None, *, mask=None, scale=None, is_causal=False, q_offset=0,
                 q_lengths=None, kv_lengths=None, block_info=None, out=None, workspace=None,
                 generic=False, flags=0, stream=None):
    """scaled_dot_product_attention(q, k, v, [bias]; mask, scale, is_causal, q_offset,
    q_lengths, kv_lengths) — is_causal is False, True or "bottom_right". `flags` takes extra
    SDPA_FLAG_* bits (e.g. the bounded-wait self-test)."""
    _check_qkv(q, k, v)
    keep = []
    p = _params(q, k, v, bias=bias, mask=mask, scale=scale, is_causal=is_causal, q_offset=q_offset,
                q_lengths=q_lengths, kv_lengths=kv_lengths, block_info=block_info,
                flags=(SDPA_FLAG_GENERIC_KERNEL if generic else 0) | flags, keep=keep)
    if out is None:
        out = torch.empty(q.shape[:3] + (v.shape[3],), dtype=q.dtype, device=q.device)
    need = _lib.sdpa_workspace_size(ctypes.byref(p))
    if need == 0:
        raise SdpaError(SDPA_ERR_INVALID_ARG, _lib.sdpa_last_error().decode())
    ws = _workspace(q.device, need, workspace)
    _check(_lib.sdpa_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), ws.ptr,
                             ws.nbytes, _stream(stream)))
    return out


def sdpa_forward_rope(q, k, v, q_positions, k_positions, bias=None, *, base=10000.0, mask=None, scale=None,
                      is_causal=False, q_offset=0, q_lengths=None, kv_lengths=None, block_info=None, out=None,
                      workspace=None, generic=False, stream=None):
    """sdpa_forward on the rotary-embedded q and k (the pair (c, c + d/2) of each row rotated by
    positions[row] * base^(-2c/d)), with q and k left as they are. q_positions: one per row of
    q, (B, Lq) or B * Lq; k_positions: one per row of k."""
    _check_qkv(q, k, v)
    keep = []
    p = _params(q, k, v, bias=bias, mask=mask, scale=scale, is_causal=is_causal, q_offset=q_offset,
                q_lengths=q_lengths, kv_lengths=kv_lengths, block_info=block_info,
                flags=SDPA_FLAG_GENERIC_KERNEL if generic else 0, keep=keep)
    qp = torch.as_tensor(q_positions, dtype=torch.int32, device=q.device).reshape(-1).contiguous()
    kp = torch.as_tensor(k_positions, dtype=torch.int32, device=q.device).reshape(-1).contiguous()
    if qp.numel() != q.shape[0] * q.shape[1] or kp.numel() != k.shape[0] * k.shape[1]:
        raise ValueError("one position per row of q and of k")
    keep += [qp, kp]
    if out is None:
        out = torch.empty(q.shape[:3] + (v.shape[3],), dtype=q.dtype, device=q.device)
    need = _lib.sdpa_rope_workspace_size(ctypes.byref(p))
    if need == 0:
        raise SdpaError(SDPA_ERR_INVALID_ARG, _lib.sdpa_last_error().decode())
    ws = _workspace(q.device, need, workspace)
    _check(_lib.sdpa_forward_rope(ctypes.byref(p), qp.data_ptr(), kp.data_ptr(), float(base), _ptr(q), _ptr(k),
                                  _ptr(v), _ptr(out), ws.ptr, ws.nbytes, _stream(stream)))
    return out


def sdpa_forward_with_weights(q, k, v, bias=None, *, mask=None, scale=None, is_causal=False, q_offset=0,
                              q_lengths=None, kv_lengths=None, block_info=None, drop_p=0.0, seed=0, out=None,
                              weights=None, workspace=None, generic=False, stream=None):
    """scaled_dot_product_attention_with_weights(q, k, v, [bias]; fdrop, mask, scale, is_causal,
    q_offset, q_lengths, kv_lengths), fdrop being dropout of probability drop_p with the
    library's counter-based generator (seed). Returns (out (B, Lq, H, dv), weights (B, H, Lq,
    Lk)), the weights after the dropout, in the page's (kv_len, q_len, nheads, batch) order."""
    _check_qkv(q, k, v)
    keep = []
    p = _params(q, k, v, bias=bias, mask=mask, scale=scale, is_causal=is_causal, q_offset=q_offset,
                q_lengths=q_lengths, kv_lengths=kv_lengths, block_info=block_info,
                flags=SDPA_FLAG_GENERIC_KERNEL if generic else 0, keep=keep)
    B, Lq, H, _ = q.shape
    if out is None:
        out = torch.empty(q.shape[:3] + (v.shape[3],), dtype=q.dtype, device=q.device)
    if weights is None:
        weights = torch.empty((B, H, Lq, k.shape[1]), dtype=q.dtype, device=q.device)
    need = _lib.sdpa_weights_workspace_size(ctypes.byref(p))
    if need == 0:
        raise SdpaError(SDPA_ERR_INVALID_ARG, _lib.sdpa_last_error().decode())
    ws = _workspace(q.device, need, workspace)
    _check(_lib.sdpa_forward_with_weights(ctypes.byref(p), float(drop_p), int(seed) & (2**64 - 1), _ptr(q),
                                          _ptr(k), _ptr(v), _ptr(out), _ptr(weights), ws.ptr, ws.nbytes,
                                          _stream(stream)))
    return out, weights


def sdpa_rope(x, positions, base=10000.0, *, out=None, stream=None):
    """Rotary position embedding of x (..., nheads, d): the pair (c, c + d/2) of each row
    rotated by positions[row] * base^(-2c/d), the rows being the leading dimensions flattened
    (positions: one per row). out may be x."""
    if not x.is_cuda or not x.is_contiguous() or x.dim() < 2 or x.dtype not in _DTYPE:
        raise ValueError("x must be a contiguous float CUDA tensor (..., nheads, d)")
    H, d = x.shape[-2], x.shape[-1]
    rows = x.numel() // (H * d) if x.numel() else 0
    pos = torch.as_tensor(positions, dtype=torch.int32, device=x.device).reshape(-1).contiguous()
    if pos.numel() != rows:
        raise ValueError(f"expected {rows} positions, got {pos.numel()}")
    if out is None:
        out = torch.empty_like(x)
    _check(_lib.sdpa_rope(_ptr(x), _ptr(out), _DTYPE[x.dtype], rows, H, d, pos.data_ptr() if rows else None,
                          float(base), _stream(stream)))
    return out


def sdpa_forward_lse(q, k, v, *, scale=None, is_causal=False, q_offset=0, q_lengths=None, kv_lengths=None,
                     out=None, workspace=None, stream=None):
    """sdpa_forward that also returns each query row's log-sum-exp (natural log, (B, H, Lq)
    float32; +inf for rows with no key or past q_lengths), for sdpa_backward(lse=...). The
    tcgen05 kernel only: bf16/fp16, head sizes 64 or 128, no bias or mask."""
    _check_qkv(q, k, v)
    keep = []
    p = _params(q, k, v, bias=None, mask=None, scale=scale, is_causal=is_causal, q_offset=q_offset,
                q_lengths=q_lengths, kv_lengths=kv_lengths, block_info=None, flags=0, keep=keep)
    if out is None:
        out = torch.empty(q.shape[:3] + (v.shape[3],), dtype=q.dtype, device=q.device)
    lse = torch.empty((q.shape[0], q.shape[2], q.shape[1]), dtype=torch.float32, device=q.device)
    need = _lib.sdpa_workspace_size(ctypes.byref(p))
    if need == 0:
        raise SdpaError(SDPA_ERR_INVALID_ARG, _lib.sdpa_last_error().decode())
    ws = _workspace(q.device, need, workspace)
    _check(_lib.sdpa_forward_lse(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), lse.data_ptr(), ws.ptr,
                                 ws.nbytes, _stream(stream)))
    return out, lse


def sdpa_backward(q, k, v, out, dout, *, mask=None, scale=None, is_causal=False, q_offset=0,
                  q_lengths=None, kv_lengths=None, block_info=None, lse=None, workspace=None, generic=False,
                  stream=None):
    """The gradient of the fused implementation for the loss sum(dout * out), where `out` is
    sdpa_forward(q, k, v; ...) with the same arguments: returns (dq, dk, dv, dscale), dscale a
    0-d float32 device tensor. Rows with no attended key and rows past q_lengths take no part.
    No bias (the page's automatic differentiation takes the materialized implementation then).
    lse: the row log-sum-exp sdpa_forward_lse returned for the same call (the tcgen05 gradient
    then does not run the forward again)."""
    _check_qkv(q, k, v)
    for n, t in (("out", out), ("dout", dout)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != q.dtype or t.shape != q.shape[:3] + (v.shape[3],):
            raise ValueError(f"{n} must be a contiguous CUDA tensor of the output's shape and dtype")
    keep = []
    p = _params(q, k, v, bias=None, mask=mask, scale=scale, is_causal=is_causal, q_offset=q_offset,
                q_lengths=q_lengths, kv_lengths=kv_lengths, block_info=block_info,
                flags=SDPA_FLAG_GENERIC_KERNEL if generic else 0, keep=keep)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dscale = torch.zeros((), dtype=torch.float32, device=q.device)
    need = _lib.sdpa_backward_workspace_size(ctypes.byref(p))
    if need == 0:
        raise SdpaError(SDPA_ERR_INVALID_ARG, _lib.sdpa_last_error().decode())
    ws = _workspace(q.device, need, workspace)
    if lse is None:
        _check(_lib.sdpa_backward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(dq),
                                  _ptr(dk), _ptr(dv), dscale.data_ptr(), ws.ptr, ws.nbytes, _stream(stream)))
    else:
        if lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous() or \
                tuple(lse.shape) != (q.shape[0], q.shape[2], q.shape[1]):
            raise ValueError("lse must be the contiguous float32 (B, H, Lq) CUDA tensor sdpa_forward_lse returned")
        _check(_lib.sdpa_backward_lse(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout),
                                      lse.data_ptr(), _ptr(dq), _ptr(dk), _ptr(dv), dscale.data_ptr(), ws.ptr,
                                      ws.nbytes, _stream(stream)))
    return dq, dk, dv, dscale


def _segments(x, device, name):
    """Segment lengths -> (device int32 tensor, host list or None). A host sequence is copied to
    the device; a device tensor stays there."""
    if isinstance(x, torch.Tensor):
        if x.dim() != 1:
            raise ValueError(f"{name} must be a vector of lengths")
        t = x.to(device=device, dtype=torch.int32).contiguous()
        return t, (None if x.is_cuda else [int(a) for a in x.tolist()])
    lens = [int(a) for a in x]
    return torch.tensor(lens, dtype=torch.int32, device=device), lens


def sdpa_forward_packed(q, k, v, q_segments, kv_segments=None, *, maxlen=None, scale=None,
                        is_causal=False, q_offset=0, q_lengths=None, kv_lengths=None, out=None,
                        workspace=None, generic=False, stream=None):
    """scaled_dot_product_attention(q, k, v; q_segments, kv_segments, maxlen, scale, is_causal,
    q_offset, q_lengths, kv_lengths) on packed sequences: q (total_q, H, dqk), k (total_kv, Hkv,
    dqk) and v (total_kv, Hkv, dv) hold the sequences one after the other; out is (total_q, H,
    dv). q_offset / q_lengths / kv_lengths take one entry per sequence. Without maxlen, lengths
    given as a device tensor are copied to the host to find it (which waits for the device)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{n} must be a contiguous 3-d CUDA tensor (total_len, heads, d)")
        if t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, k and v must share dtype and device")
    if v.shape[:2] != k.shape[:2] or k.shape[2] != q.shape[2]:
        raise ValueError("inconsistent q/k/v shapes")
    dev = q.device
    qs, q_host = _segments(q_segments, dev, "q_segments")
    keep = [qs]
    ks, kv_host = None, q_host
    if kv_segments is not None:
        ks, kv_host = _segments(kv_segments, dev, "kv_segments")
        if ks.shape != qs.shape:
            raise ValueError("kv_segments must have one entry per query segment")
        keep.append(ks)
    nseg = qs.shape[0]
    if maxlen is None:
        if q_host is None:
            q_host = [int(a) for a in qs.cpu().tolist()]
        if ks is None:
            kv_host = q_host
        elif kv_host is None:
            kv_host = [int(a) for a in ks.cpu().tolist()]
        maxlen = max(q_host + kv_host, default=0)
    p = _params(q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0), bias=None, mask=None, scale=scale,
                is_causal=is_causal, q_offset=0, q_lengths=None, kv_lengths=None, block_info=None,
                flags=SDPA_FLAG_GENERIC_KERNEL if generic else 0, keep=keep)
    if isinstance(q_offset, int):
        p.q_offset_scalar = q_offset
    else:
        t = _per_batch(q_offset, nseg, dev, "q_offset")
        keep.append(t)
        p.q_offset = t.data_ptr()
    for name, val in (("q_lengths", q_lengths), ("kv_lengths", kv_lengths)):
        t = _per_batch(val, nseg, dev, name)
        if t is not None:
            keep.append(t)
            setattr(p, name, t.data_ptr())
    seg = PackedSegments(nseg, int(maxlen), qs.data_ptr(), None if ks is None else ks.data_ptr())
    if out is None:
        out = torch.empty(q.shape[:2] + (v.shape[2],), dtype=q.dtype, device=dev)
    need = _lib.sdpa_packed_workspace_size(ctypes.byref(p), ctypes.byref(seg))
    if need == 0:
        raise SdpaError(SDPA_ERR_INVALID_ARG, _lib.sdpa_last_error().decode())
    ws = _workspace(dev, need, workspace)
    _check(_lib.sdpa_forward_packed(ctypes.byref(p), ctypes.byref(seg), _ptr(q), _ptr(k), _ptr(v),
                                    _ptr(out), ws.ptr, ws.nbytes, _stream(stream)))
    return out


def sdpa_decode_with_cache(q, k_new, v_new, k_cache, v_cache, cache_index, *, scale=None,
                           out=None, workspace=None, generic=False, stream=None):
    """Writes k_new/v_new (B, n_new, Hkv, d) into the caches (B, capacity, Hkv, d) at
    cache_index[b], then attends q (B, n_new, H, d) with :bottom_right alignment over
    cache_index[b] + n_new keys."""
    _check_qkv(q, k_cache, v_cache)
    idx = _per_batch(cache_index, q.shape[0], q.device, "cache_index")
    keep = [idx]
    p = _params(q, k_cache, v_cache, bias=None, mask=None, scale=scale, is_causal="bottom_right",
                q_offset=0, q_lengths=None, kv_lengths=None, block_info=None,
                flags=SDPA_FLAG_GENERIC_KERNEL if generic else 0, keep=keep)
    if out is None:
        out = torch.empty(q.shape[:3] + (v_cache.shape[3],), dtype=q.dtype, device=q.device)
    need = _lib.sdpa_workspace_size(ctypes.byref(p))
    if need == 0:
        raise SdpaError(SDPA_ERR_INVALID_ARG, _lib.sdpa_last_error().decode())
    ws = _workspace(q.device, need, workspace)
    _check(_lib.sdpa_decode_with_cache(ctypes.byref(p), _ptr(q), _ptr(k_new), _ptr(v_new),
                                       _ptr(k_cache), _ptr(v_cache), idx.data_ptr(), _ptr(out),
                                       ws.ptr, ws.nbytes, _stream(stream)))
    return out


def cache_update_at_index(k_cache, v_cache, k_new, v_new, index, *, workspace=None, stream=None):
    """Writes k_new/v_new (B, n_new, Hkv, d) into k_cache/v_cache (B, capacity, Hkv, d) at rows
    index[b] .. index[b] + n_new - 1, in place."""
    ref = k_cache if k_cache is not None else v_cache
    B, cap, Hkv, d = ref.shape
    n_new = (k_new if k_new is not None else v_new).shape[1]
    idx = _per_batch(index, B, ref.device, "index")
    ws = _workspace(ref.device, 256, workspace)
    _check(_lib.cache_update_at_index(_ptr(k_cache), _ptr(v_cache), _ptr(k_new), _ptr(v_new),
                                      _DTYPE[ref.dtype], d, Hkv, n_new, cap, B, idx.data_ptr(),
                                      ws.ptr, _stream(stream)))


class BlockMaskInfo:
    """Device-resident classification of a boolean mask (owns its buffer)."""

    def __init__(self, buf, struct, mask_shape):
        self.buf = buf
        self.struct = struct
        self.mask_shape = mask_shape

    def _view(self, ptr, dtype, shape):
        n = 1
        for s in shape:
            n *= s
        off = ptr - self.buf.data_ptr()
        itemsize = torch.empty((), dtype=dtype).element_size()
        return self.buf[off:off + n * itemsize].view(dtype).view(*shape)

    def arrays(self):
        s = self.struct
        words = s.bk // 32
        return dict(
            cls=self._view(s.block_class, torch.uint8, (s.nheads, s.nqb, s.nkb)),
            count=self._view(s.row_count, torch.int32, (s.nheads, s.nqb)),
            list=self._view(s.row_list, torch.int32, (s.nheads, s.nqb, s.nkb)),
            bits=self._view(s.partial_bits, torch.int32, (s.nheads, s.nqb, s.nkb, s.bq, words)))


def build_block_mask_info(mask, bq: int = 128, bk: int = 128, *, stream=None) -> BlockMaskInfo:
    """Classifies the bq x bk blocks of a boolean mask of row-major shape (H, Lq, Lk) (the page's
    (kv_len, q_len, nheads)); its key axis must be contiguous."""
    if mask.dim() != 3 or mask.dtype not in (torch.bool, torch.uint8) or not mask.is_cuda:
        raise ValueError("mask must be a 3-d bool/uint8 CUDA tensor (H, Lq, Lk)")
    H, Lq, Lk = mask.shape
    need = _lib.build_block_mask_info_size(H, Lq, Lk, bq, bk)
    if need == 0:
        raise SdpaError(SDPA_ERR_INVALID_ARG, "invalid block mask sizes")
    raw = torch.empty(need + 256, dtype=torch.uint8, device=mask.device)
    off = (-raw.data_ptr()) % 256
    buf = raw[off:off + need]
    st = BlockMaskInfoStruct()
    strides = (ctypes.c_int64 * 3)(mask.stride(2), mask.stride(1), mask.stride(0))
    _check(_lib.build_block_mask_info(mask.data_ptr(), strides, H, Lq, Lk, bq, bk, buf.data_ptr(),
                                      need, ctypes.byref(st), _stream(stream)))
    info = BlockMaskInfo(buf, st, (H, Lq, Lk))
    info._raw = raw
    return info


__all__ = ["sdpa_forward", "sdpa_forward_lse", "sdpa_forward_packed", "sdpa_forward_rope", "sdpa_forward_with_weights", "sdpa_rope", "sdpa_backward", "sdpa_decode_with_cache", "cache_update_at_index",
           "build_block_mask_info", "BlockMaskInfo", "Workspace", "read_device_status",
           "last_kernel", "SdpaError", "lib"]
