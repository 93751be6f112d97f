"""GPU parity of the rotary position embedding (rotary embeddings on query and key, from the
Keras thread on MultiHeadAttention; the form used is the pair (c, c + d/2) rotated by
position * base^(-2c/d)) against the CPU oracle, through the C ABI: the standalone pass, the
attention call with the embedding folded in (sdpa_forward_rope), and sliding-window caches
addressed through q_offset (the NNlib entry's q_offset argument)."""
import numpy as np
import pytest
import torch

import oracle
import sdpa_inputs as si
from parity import assert_matches, f64

pytestmark = pytest.mark.gpu

sdpa = pytest.importorskip("head_scaled_dot_sdpa_b200")
DEV = "cuda"
TOL = {torch.float32: 1e-5, torch.float16: 1e-2, torch.bfloat16: 1e-2}


def assert_close(got, want, tol, what):
    g, w = f64(got), f64(want)
    err = np.abs(g - w) / np.maximum(1.0, np.abs(w))
    assert err.max() <= tol, f"{what}: error {err.max():.3e} > {tol:g}"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("shape", [(7, 3, 2), (130, 8, 64), (513, 4, 128), (33, 2, 80)])
def test_rope_matches_the_oracle(dtype, shape):
    rows, H, d = shape
    rng = np.random.Generator(np.random.PCG64(rows + d))
    x = si.normal(rng, shape, {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}[dtype])
    pos = rng.integers(-1000, 200000, size=rows)
    out = sdpa.sdpa_rope(x.to(DEV), torch.from_numpy(pos).to(torch.int32))
    assert_close(out, oracle.rope(f64(x), pos), TOL[dtype], f"rope {shape} {dtype}")


def test_rope_in_place_on_a_padded_batch():
    """A (batch, seq, heads, d) array flattens to batch * seq rows; the call may write in place."""
    rng = np.random.Generator(np.random.PCG64(3))
    x = si.normal(rng, (2, 100, 8, 128), "bf16")
    pos = np.concatenate([np.arange(100), 4000 + np.arange(100)])
    xd = x.to(DEV)
    sdpa.sdpa_rope(xd, torch.from_numpy(pos).to(torch.int32), out=xd)
    want = oracle.rope(f64(x).reshape(200, 8, 128), pos).reshape(2, 100, 8, 128)
    assert_close(xd, want, 1e-2, "in place")


def _rounded(x64, dtype):
    """The oracle's rotated array rounded to the input type, as the rotated q / k are held."""
    return f64(torch.from_numpy(x64).to(dtype))


FUSED = [
    # B, Lq, Lk, H, Hkv, D, causal
    (2, 300, 300, 8, 2, 128, True),
    (1, 200, 333, 4, 4, 64, "bottom_right"),
    (2, 129, 257, 6, 3, 128, False),
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("shape", FUSED, ids=lambda s: "x".join(map(str, s)))
def test_fused_rope_prefill_matches_the_oracle(dtype, shape):
    """sdpa_forward_rope = attention on rope(q), rope(k): the tcgen05 kernel rotates its Q tiles
    in shared memory (several tiles and a ragged tail), the keys are rotated once."""
    B, Lq, Lk, H, Hkv, D, causal = shape
    rng = np.random.Generator(np.random.PCG64(Lq + Lk + D))
    name = {torch.float16: "f16", torch.bfloat16: "bf16"}[dtype]
    q = si.normal(rng, (B, Lq, H, D), name)
    k = si.normal(rng, (B, Lk, Hkv, D), name)
    v = si.normal(rng, (B, Lk, Hkv, D), name)
    qpos = rng.integers(0, 50000, size=(B, Lq)).astype(np.int32)
    kpos = rng.integers(0, 50000, size=(B, Lk)).astype(np.int32)
    out = sdpa.sdpa_forward_rope(q.to(DEV), k.to(DEV), v.to(DEV), torch.from_numpy(qpos), torch.from_numpy(kpos),
                                 is_causal=causal)
    assert sdpa.last_kernel() == "prefill_tcgen05_rope"
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    qr = _rounded(oracle.rope(f64(q).reshape(B * Lq, H, D), qpos.ravel()), dtype).reshape(B, Lq, H, D)
    kr = _rounded(oracle.rope(f64(k).reshape(B * Lk, Hkv, D), kpos.ravel()), dtype).reshape(B, Lk, Hkv, D)
    want = oracle.sdpa_forward(qr, kr, f64(v), is_causal=causal)
    assert_matches(out, want, 1e-2, f"fused rope {shape}")


def test_fused_rope_fp32_takes_the_simt_kernel():
    rng = np.random.Generator(np.random.PCG64(77))
    B, Lq, Lk, H, Hkv, D = 1, 33, 50, 4, 2, 32
    q, k, v = (si.normal(rng, s, "f32") for s in [(B, Lq, H, D), (B, Lk, Hkv, D), (B, Lk, Hkv, D)])
    qpos, kpos = np.arange(Lq, dtype=np.int32) + 17, np.arange(Lk, dtype=np.int32)
    out = sdpa.sdpa_forward_rope(q.to(DEV), k.to(DEV), v.to(DEV), torch.from_numpy(qpos), torch.from_numpy(kpos),
                                 is_causal=True, q_offset=17)
    assert sdpa.last_kernel() == "generic_simt"
    qr = oracle.rope(f64(q).reshape(Lq, H, D), qpos).reshape(B, Lq, H, D)
    kr = oracle.rope(f64(k).reshape(Lk, Hkv, D), kpos).reshape(B, Lk, Hkv, D)
    want = oracle.sdpa_forward(_rounded(qr, torch.float32), _rounded(kr, torch.float32), f64(v), is_causal=True,
                               q_offset=17)
    assert_matches(out, want, 1e-5, "fused rope fp32")


def _rotated_sequence(rng, T, H, Hkv, D):
    """A sequence of T tokens whose keys (and queries) are rotary-embedded at their absolute
    positions, as a cache holds them."""
    q = si.normal(rng, (1, T, H, D), "bf16")
    k = si.normal(rng, (1, T, Hkv, D), "bf16")
    v = si.normal(rng, (1, T, Hkv, D), "bf16")
    pos = torch.arange(T, dtype=torch.int32)
    qr = sdpa.sdpa_rope(q.to(DEV), pos).cpu()
    kr = sdpa.sdpa_rope(k.to(DEV), pos).cpu()
    return qr, kr, v


def test_sliding_window_ring_cache_decode():
    """A sliding-window KV cache as a ring of W slots (token p in slot p % W) holds the last W
    keys. The query of the newest token attends all of them: with q_offset counting the keys
    kept (W - 1 before it), not the absolute position (the NNlib entry's q_offset argument).
    Checked against the oracle on the whole sequence with the window as an explicit mask."""
    rng = np.random.Generator(np.random.PCG64(21))
    T, W, H, Hkv, D = 1000, 256, 8, 2, 128
    qr, kr, v = _rotated_sequence(rng, T, H, Hkv, D)
    window = np.arange(T - W, T)
    ring = np.empty(W, dtype=np.int64)
    ring[window % W] = window  # slot -> token
    k_ring, v_ring = kr[:, ring], v[:, ring]
    q_last = qr[:, T - 1:T]
    out = sdpa.sdpa_forward(q_last.to(DEV), k_ring.to(DEV), v_ring.to(DEV), is_causal=True, q_offset=W - 1)
    mask = np.zeros((1, 1, 1, T), dtype=bool)
    mask[..., T - W:] = True
    want = oracle.sdpa_forward(f64(q_last), f64(kr), f64(v), mask=mask, is_causal=True, q_offset=T - 1)
    assert_matches(out, want, 1e-2, "ring cache decode")


def test_sliding_window_chunked_prefill():
    """A chunk of n new queries after a cache that kept only the last W keys: the buffer holds
    those W keys and the n new ones, and q_offset = W counts the kept keys before the chunk.
    Query t (absolute position P + t) then attends keys P - W .. P + t of the whole sequence."""
    rng = np.random.Generator(np.random.PCG64(22))
    P, W, n, H, Hkv, D = 700, 192, 64, 8, 2, 128
    T = P + n
    qr, kr, v = _rotated_sequence(rng, T, H, Hkv, D)
    keep = np.arange(P - W, T)
    out = sdpa.sdpa_forward(qr[:, P:].to(DEV), kr[:, keep].to(DEV), v[:, keep].to(DEV), is_causal=True, q_offset=W)
    mask = np.zeros((1, 1, n, T), dtype=bool)
    mask[..., P - W:] = True
    want = oracle.sdpa_forward(f64(qr[:, P:]), f64(kr), f64(v), mask=mask, is_causal=True, q_offset=P)
    assert_matches(out, want, 1e-2, "sliding-window chunk")


def test_fused_rope_with_a_mask_rotates_into_the_workspace():
    """With a mask the queries are rotated into the workspace and the tcgen05 kernel takes the
    rotated arrays with its dense-mask variant."""
    rng = np.random.Generator(np.random.PCG64(78))
    B, Lq, Lk, H, Hkv, D = 1, 160, 192, 4, 2, 128
    q, k, v = (si.normal(rng, s, "bf16") for s in [(B, Lq, H, D), (B, Lk, Hkv, D), (B, Lk, Hkv, D)])
    qpos, kpos = rng.integers(0, 9000, size=B * Lq).astype(np.int32), rng.integers(0, 9000, size=B * Lk).astype(np.int32)
    mask = torch.from_numpy(rng.random((H, Lq, Lk)) < 0.7)
    out = sdpa.sdpa_forward_rope(q.to(DEV), k.to(DEV), v.to(DEV), torch.from_numpy(qpos), torch.from_numpy(kpos),
                                 mask=mask.to(DEV))
    assert sdpa.last_kernel() == "prefill_tcgen05"
    qr = _rounded(oracle.rope(f64(q).reshape(Lq, H, D), qpos), torch.bfloat16).reshape(B, Lq, H, D)
    kr = _rounded(oracle.rope(f64(k).reshape(Lk, Hkv, D), kpos), torch.bfloat16).reshape(B, Lk, Hkv, D)
    want = oracle.sdpa_forward(qr, kr, f64(v), mask=mask.numpy()[None])
    assert_matches(out, want, 1e-2, "rope + mask")
