"""GPU parity of scaled_dot_product_attention_with_weights with dropout as fdrop (the NNlib
entry's "See also" and its fdrop argument) against the CPU oracle, through the C ABI: the
output and the materialized weights, the dropout decisions bit for bit (both sides draw the
same counter-based generator and compare in double).

Tolerance. The forward bounds (1e-5 fp32, 1e-2 bf16/fp16) are taken relative to the larger of
1 and the oracle's magnitude: |got - want| <= tol * max(1, |want|). Rows that attend a few
keys, scaled by the dropout's 1/(1 - p), have outputs of magnitude 2 to 5. There the 16-bit
output's own rounding, half an ulp = 2^-9 |x| for bf16, already reaches 1e-2 in absolute
terms. On a B200 the fp32 SIMT kernel's output was off by exactly that (0.0156 at 4.14)."""
import numpy as np
import pytest
import torch

import oracle
import sdpa_inputs as si
from parity import f64

pytestmark = pytest.mark.gpu

sdpa = pytest.importorskip("head_scaled_dot_sdpa_b200")
DEV = "cuda"
NAMES = {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}
TOL = {torch.float32: 1e-5, torch.float16: 1e-2, torch.bfloat16: 1e-2}


def assert_matches(got, want, tol, what):
    """NaN exactly where the oracle has NaN; elsewhere |got - want| <= tol * max(1, |want|)."""
    g, w = f64(got), f64(want)
    assert g.shape == w.shape, f"{what}: shape {g.shape} vs {w.shape}"
    gn, wn = np.isnan(g), np.isnan(w)
    assert (gn == wn).all(), f"{what}: NaN pattern differs at {np.argwhere(gn != wn)[:5].tolist()}"
    ok = ~wn
    if ok.any():
        err = np.abs(g[ok] - w[ok]) / np.maximum(1.0, np.abs(w[ok]))
        i = int(np.argmax(err))
        assert err[i] <= tol, f"{what}: error {err[i]:.3e} > {tol:g} (oracle {w[ok][i]:.4f}, got {g[ok][i]:.4f})"


def _inputs(seed, B, Lq, Lk, H, Hkv, D, Dv, dtype):
    rng = np.random.Generator(np.random.PCG64(seed))
    n = NAMES[dtype]
    return (si.normal(rng, (B, Lq, H, D), n), si.normal(rng, (B, Lk, Hkv, D), n),
            si.normal(rng, (B, Lk, Hkv, Dv), n))


def check(q, k, v, what, bias=None, kernel=None, **kw):
    dev = lambda t: None if t is None else t.to(DEV)
    out, w = sdpa.sdpa_forward_with_weights(dev(q), dev(k), dev(v), dev(bias), **kw)
    if kernel:
        assert sdpa.last_kernel() == kernel
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    okw = {a: b for a, b in kw.items() if a not in ("block_info", "generic")}
    if "mask" in okw:
        okw["mask"] = okw["mask"].cpu().numpy()
    want_o, want_w = oracle.sdpa_forward_with_weights(f64(q), f64(k), f64(v), None if bias is None else f64(bias), **okw)
    tol = TOL[q.dtype]
    assert_matches(w, want_w, tol, f"{what} weights")
    assert_matches(out, want_o, tol, f"{what} out")
    if kw.get("drop_p", 0.0) > 0:
        g, ww = f64(w), want_w
        assert ((g == 0) == (ww == 0)).all(), f"{what}: dropout pattern differs"


def kernel_for(q, v, generic=False):
    tiles = q.dtype in (torch.bfloat16, torch.float16) and q.shape[-1] == v.shape[-1] in (64, 128)
    return "weights_mma" if tiles and not generic else "weights_simt"


SHAPES = [
    # B, Lq, Lk, H, Hkv, D, Dv
    (2, 37, 45, 4, 2, 64, 64),
    (1, 130, 200, 2, 1, 128, 128),
    (2, 64, 33, 3, 3, 40, 24),
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True, "bottom_right"])
@pytest.mark.parametrize("drop_p", [0.0, 0.25])
def test_weights_shapes(dtype, shape, causal, drop_p):
    B, Lq, Lk, H, Hkv, D, Dv = shape
    q, k, v = _inputs(Lq + Lk + D, B, Lq, Lk, H, Hkv, D, Dv, dtype)
    check(q, k, v, f"{shape} causal={causal} p={drop_p}", kernel=kernel_for(q, v), is_causal=causal,
          drop_p=drop_p, seed=11)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_weights_bias_mask_lengths(dtype):
    """A broadcast bias, a dense mask, per-batch offsets and lengths, a sequence with no key
    (NaN weights and output) and padding rows (zeros)."""
    q, k, v = _inputs(3, 3, 50, 70, 4, 2, 64, 64, dtype)
    rng = np.random.Generator(np.random.PCG64(4))
    bias = torch.from_numpy(rng.standard_normal((4, 50, 70)).astype(np.float32)).to(dtype)
    mask = torch.from_numpy(rng.random((4, 50, 70)) < 0.8).to(DEV)
    check(q, k, v, "bias+mask+lengths", bias=bias, mask=mask, is_causal=True, q_offset=[20, -5, 0],
          q_lengths=[50, 31, 12], kv_lengths=[70, 40, 0], drop_p=0.1, seed=5)


def test_weights_simt_forced_and_block_info():
    q, k, v = _inputs(6, 1, 300, 260, 2, 2, 128, 128, torch.bfloat16)
    check(q, k, v, "forced SIMT", kernel="weights_simt", generic=True, is_causal=True, drop_p=0.2, seed=1)
    w = si.scaled(si.BLOCK_SPARSE, nheads=2, nkvheads=2, q_len=300, kv_len=260, block=128)
    mask = si.mask_device(w, si.block_classes(w), DEV)
    info = sdpa.build_block_mask_info(mask)
    check(q, k, v, "block info", kernel="weights_mma", mask=mask, block_info=info)


def test_weights_without_dropout_match_the_fused_output():
    """With p = 0 the output is the fused implementation's (up to the rounding of the weights)."""
    q, k, v = _inputs(9, 2, 256, 256, 8, 2, 128, 128, torch.bfloat16)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out, _ = sdpa.sdpa_forward_with_weights(qd, kd, vd, is_causal=True)
    fused = sdpa.sdpa_forward(qd, kd, vd, is_causal=True)
    assert_matches(out, f64(fused), 1e-2, "with weights vs fused")
