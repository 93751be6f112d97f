"""GPU parity of the fused gradient (dq, dk, dv, dscale; paragraph "Fused implementation" of
NNlib.scaled_dot_product_attention) against the CPU oracle's gradient, through the C ABI.

Tolerance. A gradient element sums many terms of the size of the forward's outputs, so the
forward bounds (1e-5 for fp32, 1e-2 for bf16/fp16, as max-abs error on O(1) values) are taken
relative to the larger of 1 and the oracle's magnitude: |got - want| <= tol * max(1, |want|).
For 16-bit inputs two roundings enter besides the fp32 arithmetic. The first is the rounding
of dq/dk/dv to the input type, a relative 2^-9. The second is delta = dout . out taken from
the 16-bit forward output, which perturbs every weight's gradient by the relative rounding of
out. Both stay well inside 1e-2.
"""
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


def assert_close_rel(got, want, tol, what):
    g, w = f64(got), f64(want)
    assert g.shape == w.shape, f"{what}: shape {g.shape} vs {w.shape}"
    assert np.isfinite(g).all(), f"{what}: non-finite gradient"
    err = np.abs(g - w) / np.maximum(1.0, np.abs(w))
    i = np.unravel_index(int(np.argmax(err)), err.shape)
    assert err[i] <= tol, f"{what}: relative error {err[i]:.3e} > {tol:g} at {i} (oracle {w[i]:.5f}, got {g[i]:.5f})"


def _inputs(seed, B, Lq, Lk, H, Hkv, D, Dv, dtype):
    rng = np.random.Generator(np.random.PCG64(seed))
    n = NAMES[dtype]
    return (si.normal(rng, (B, Lq, H, D), n), si.normal(rng, (B, Lk, Hkv, D), n),
            si.normal(rng, (B, Lk, Hkv, Dv), n), si.normal(rng, (B, Lq, H, Dv), n))


def expected_kernel(q, v, generic=False, masked=False):
    """16-bit types: head_dim = v_head_dim = 128 without a mask on tcgen05, 64 or 128 on mma.sync
    tiles; SIMT otherwise."""
    tiles = q.dtype in (torch.bfloat16, torch.float16) and q.shape[-1] == v.shape[-1] in (64, 128)
    if generic or not tiles:
        return "backward_simt"
    return "backward_tcgen05" if q.shape[-1] == 128 and not masked else "backward_mma"


def check(q, k, v, dout, what, generic=False, **kw):
    """Forward on the GPU, then the gradient on the GPU, against the oracle's gradient."""
    dt = q.dtype
    qd, kd, vd, dd = (t.to(DEV) for t in (q, k, v, dout))
    out = sdpa.sdpa_forward(qd, kd, vd, **kw)
    dq, dk, dv, ds = sdpa.sdpa_backward(qd, kd, vd, out, dd, generic=generic, **kw)
    assert sdpa.last_kernel() == expected_kernel(q, v, generic, masked="mask" in kw or "block_info" in kw)
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    okw = {a: b for a, b in kw.items() if a != "block_info"}
    if "mask" in okw:
        okw["mask"] = okw["mask"].cpu().numpy()
    wq, wk, wv, wds = oracle.sdpa_backward(f64(q), f64(k), f64(v), f64(dout), **okw)
    tol = TOL[dt]
    assert_close_rel(dq, wq, tol, f"{what} dq")
    assert_close_rel(dk, wk, tol, f"{what} dk")
    assert_close_rel(dv, wv, tol, f"{what} dv")
    # dscale sums one term per query row (q_i . dq_i / scale): its error is relative to the sum
    # of those terms' magnitudes
    scale = kw.get("scale") or 1.0 / np.sqrt(q.shape[-1])
    mag = float(np.abs((f64(q) * wq).sum(axis=-1)).sum()) / scale
    assert abs(float(ds) - wds) <= tol * max(1.0, mag), f"{what} dscale {float(ds)} vs {wds} (terms {mag:.3f})"


SHAPES = [
    # B, Lq, Lk, H, Hkv, D, Dv: ragged tails of the 64-query, 64-key and 32-query tiles,
    # several tiles, GQA groups of 1 to 4
    (2, 37, 45, 4, 2, 64, 64),
    (1, 130, 200, 2, 1, 128, 128),
    (2, 64, 33, 3, 3, 40, 24),
    (1, 200, 131, 8, 2, 128, 128),
    (2, 97, 97, 3, 1, 64, 64),
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True, "bottom_right"])
def test_backward_shapes(dtype, shape, causal):
    B, Lq, Lk, H, Hkv, D, Dv = shape
    q, k, v, dout = _inputs(Lq + Lk + D, B, Lq, Lk, H, Hkv, D, Dv, dtype)
    check(q, k, v, dout, f"{shape} causal={causal}", is_causal=causal)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("causal", [False, True, "bottom_right"])
def test_backward_tcgen05_gqa_tiles(dtype, causal):
    """The tcgen05 gradient with several query and key tiles per unit, ragged tails on both,
    unequal lengths and GQA groups of 4."""
    q, k, v, dout = _inputs(31, 2, 300, 389, 8, 2, 128, 128, dtype)
    check(q, k, v, dout, f"tcgen05 gqa causal={causal}", is_causal=causal)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_simt_forced(causal):
    """The SIMT kernels on a shape the tiles also take, so both paths stay covered."""
    q, k, v, dout = _inputs(8, 1, 100, 90, 4, 2, 128, 128, torch.bfloat16)
    check(q, k, v, dout, f"forced SIMT causal={causal}", generic=True, is_causal=causal)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_backward_lengths_offsets_and_empty_rows(dtype):
    """Per-batch q_offset, q_lengths and kv_lengths, with a sequence of no keys (NaN rows, no
    part in the gradient) and padding rows."""
    q, k, v, dout = _inputs(5, 3, 50, 70, 4, 2, 64, 64, dtype)
    check(q, k, v, dout, "lengths", is_causal=True, q_offset=[20, -5, 0], q_lengths=[50, 31, 12],
          kv_lengths=[70, 40, 0])
    if dtype != torch.float32:  # the same on the tcgen05 kernels (head_dim 128), tiles ragged
        q, k, v, dout = _inputs(7, 3, 200, 270, 4, 2, 128, 128, dtype)
        check(q, k, v, dout, "lengths tcgen05", is_causal=True, q_offset=[20, -5, 0], q_lengths=[200, 131, 12],
              kv_lengths=[270, 140, 0])


def test_backward_mask_and_block_info():
    """A dense boolean mask, and the same mask through its block classification."""
    w = si.scaled(si.BLOCK_SPARSE, nheads=2, nkvheads=2, q_len=300, kv_len=260, block=128)
    mask = si.mask_device(w, si.block_classes(w), DEV)
    q, k, v, dout = _inputs(6, 1, 300, 260, 2, 2, 128, 128, torch.bfloat16)
    check(q, k, v, dout, "dense mask", mask=mask)
    info = sdpa.build_block_mask_info(mask)
    check(q, k, v, dout, "block info", mask=mask, block_info=info)


def test_backward_full_size_sampled():
    """The causal GQA prefill workload at its full size (bf16, batch 4, 32 query / 8 key-value
    heads, head_dim 128, 2048 positions), launched as the benchmark launches it. Two
    (batch, key/value head) groups are checked against the oracle run on that group alone:
    its four query heads' dq, and the group's dk and dv."""
    w = si.CAUSAL_GQA_PREFILL
    q, k, v = si.qkv(w)
    dout = si.normal(si.rng_for(w.seed + 7), tuple(q.shape), w.dtype)
    qd, kd, vd, dd = (t.to(DEV) for t in (q, k, v, dout))
    out = sdpa.sdpa_forward(qd, kd, vd, is_causal=True)
    dq, dk, dv, _ = sdpa.sdpa_backward(qd, kd, vd, out, dd, is_causal=True)
    assert sdpa.last_kernel() == "backward_tcgen05"
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    g = w.nheads // w.nkvheads
    for b, kvh in ((0, 0), (3, 5)):
        hs = slice(kvh * g, (kvh + 1) * g)
        wq, wk, wv, _ = oracle.sdpa_backward(f64(q[b:b + 1, :, hs]), f64(k[b:b + 1, :, kvh:kvh + 1]),
                                             f64(v[b:b + 1, :, kvh:kvh + 1]), f64(dout[b:b + 1, :, hs]),
                                             is_causal=True)
        assert_close_rel(dq[b:b + 1, :, hs], wq, 1e-2, f"dq b={b} kv head {kvh}")
        assert_close_rel(dk[b:b + 1, :, kvh:kvh + 1], wk, 1e-2, f"dk b={b} kv head {kvh}")
        assert_close_rel(dv[b:b + 1, :, kvh:kvh + 1], wv, 1e-2, f"dv b={b} kv head {kvh}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_forward_lse_and_backward_from_it(dtype):
    """sdpa_forward_lse's row log-sum-exp against the oracle's (natural log, +inf for rows with
    no key or past q_lengths), and the gradient that takes it instead of running the forward
    again, against the oracle's gradient."""
    q, k, v, dout = _inputs(17, 3, 200, 270, 4, 2, 128, 128, dtype)
    kw = dict(is_causal=True, q_offset=[20, -5, 0], q_lengths=[200, 131, 12], kv_lengths=[270, 140, 0])
    qd, kd, vd, dd = (t.to(DEV) for t in (q, k, v, dout))
    out, lse = sdpa.sdpa_forward_lse(qd, kd, vd, **kw)
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    want_o, want_lse = oracle.sdpa_forward_lse(f64(q), f64(k), f64(v), **kw)
    got = lse.cpu().double().numpy()
    assert np.array_equal(np.isinf(got), np.isinf(want_lse)), "lse: +inf pattern differs"
    fin = np.isfinite(want_lse)
    assert np.abs(got[fin] - want_lse[fin]).max() <= 1e-4
    fwd = sdpa.sdpa_forward(qd, kd, vd, **kw)
    assert torch.equal(torch.nan_to_num(out), torch.nan_to_num(fwd))  # the same output
    dq, dk, dv, ds = sdpa.sdpa_backward(qd, kd, vd, out, dd, lse=lse, **kw)
    assert sdpa.last_kernel() == "backward_tcgen05"
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    wq, wk, wv, wds = oracle.sdpa_backward(f64(q), f64(k), f64(v), f64(dout), **kw)
    for name, g, w in (("dq", dq, wq), ("dk", dk, wk), ("dv", dv, wv)):
        assert_close_rel(g, w, 1e-2, f"lse path {name}")
    mag = float(np.abs((f64(q) * wq).sum(axis=-1)).sum()) * np.sqrt(q.shape[-1])
    assert abs(float(ds) - wds) <= 1e-2 * max(1.0, mag)
