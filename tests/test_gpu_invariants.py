"""Invariants of the definition checked on the CUDA path itself (the oracle's pins, run again
on the GPU): properties that hold at any size, so they also cover sizes the oracle is too slow
for. NNlib.scaled_dot_product_attention on the Flux.jl page "Neural Network primitives from
NNlib.jl", sections "Arguments" and "Examples". Named to run after the parity tests."""
import numpy as np
import pytest
import torch

import sdpa_inputs as si
from parity import f64

pytestmark = pytest.mark.gpu

sdpa = pytest.importorskip("head_scaled_dot_sdpa_b200")
DEV = "cuda"


def assert_matches(got, want, tol, what):
    """Two CUDA results of the same quantity: NaN in the same places, elsewhere
    |got - want| <= tol * max(1, |want|) (one 16-bit ulp above 2 is more than 1e-2)."""
    g, w = f64(got), f64(want)
    assert g.shape == w.shape and (np.isnan(g) == np.isnan(w)).all(), what
    ok = ~np.isnan(w)
    err = np.abs(g[ok] - w[ok]) / np.maximum(1.0, np.abs(w[ok]))
    assert err.max(initial=0.0) <= tol, f"{what}: error {err.max():.3e} > {tol:g}"


def _qkv(seed, B, Lq, Lk, H, Hkv, D, dtype=torch.bfloat16):
    rng = np.random.Generator(np.random.PCG64(seed))
    n = {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}[dtype]
    return tuple(si.normal(rng, s, n).to(DEV) for s in ((B, Lq, H, D), (B, Lk, Hkv, D), (B, Lk, Hkv, D)))


def test_constant_values_give_constant_output():
    """The weights of a row sum to one: with every value equal to 1 the output is 1."""
    q, k, _ = _qkv(1, 2, 1000, 3000, 16, 4, 128)
    v = torch.ones_like(k)
    out = sdpa.sdpa_forward(q, k, v, is_causal="bottom_right")
    assert (out.float() - 1).abs().max().item() <= 1e-2


def test_gqa_equals_repeated_heads():
    """Argument sharing of key/value heads (the GQA paragraph): query head h reads key/value
    head h // (nheads / nkvheads), the same as repeating each key/value head over its group."""
    q, k, v = _qkv(2, 2, 700, 900, 32, 8, 128)
    a = sdpa.sdpa_forward(q, k, v, is_causal=True)
    b = sdpa.sdpa_forward(q, k.repeat_interleave(4, dim=2).contiguous(), v.repeat_interleave(4, dim=2).contiguous(),
                          is_causal=True)
    assert_matches(a, f64(b), 1e-2, "GQA vs repeated heads")


def test_kv_lengths_equal_truncation():
    """Argument kv_lengths: keys past the length are not attended, the same as dropping them."""
    q, k, v = _qkv(3, 1, 600, 2000, 8, 8, 64, torch.float16)
    a = sdpa.sdpa_forward(q, k, v, kv_lengths=[1333])
    b = sdpa.sdpa_forward(q, k[:, :1333].contiguous(), v[:, :1333].contiguous())
    assert_matches(a, f64(b), 1e-2, "kv_lengths vs truncation")


def test_printed_bottom_right_example_at_scale():
    """Example "decoding with a KV cache": :bottom_right with kv_lengths equals is_causal with
    q_offset = kv_lengths - q_len, here with 128 new queries and 64 heads."""
    q, k, v = _qkv(4, 4, 128, 4096, 64, 8, 128)
    kvl = [1000, 2300, 3300, 4096]
    a = sdpa.sdpa_forward(q, k, v, is_causal="bottom_right", kv_lengths=kvl)
    b = sdpa.sdpa_forward(q, k, v, is_causal=True, q_offset=[n - 128 for n in kvl], kv_lengths=kvl)
    assert_matches(a, f64(b), 1e-3, "bottom_right vs q_offset")


def test_scale_equivalence():
    """Argument scale: sdpa(a q; scale s) = sdpa(q; scale a s)."""
    q, k, v = _qkv(5, 2, 300, 300, 4, 2, 128, torch.float32)
    a = sdpa.sdpa_forward(q * 2, k, v, scale=0.05)
    b = sdpa.sdpa_forward(q, k, v, scale=0.1)
    assert_matches(a, f64(b), 1e-5, "scale equivalence")
