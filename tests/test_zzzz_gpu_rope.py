"""GPU parity of the rotary position embedding (rotary embeddings on query and key, from the
Keras thread on MultiHeadAttention; the form used is the pair (c, c + d/2) rotated by
position * base^(-2c/d)) against the CPU oracle, through the C ABI. Named to run last."""
import numpy as np
import pytest
import torch

import oracle
import sdpa_inputs as si
from parity import f64

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
