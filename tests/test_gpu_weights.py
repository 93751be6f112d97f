"""GPU parity of scaled_dot_product_attention_with_weights with dropout as fdrop (the NNlib
entry's "See also" and its fdrop argument) against the CPU oracle, through the C ABI: the
output and the materialized weights, the dropout decisions bit for bit (both sides draw the
same counter-based generator and compare in double).

Tolerance. The forward bounds (1e-5 fp32, 1e-2 bf16/fp16) in absolute terms, applied as in
the other parity tests to the value before the 16-bit output's own rounding (parity.py): a
16-bit element passes when |got - want| <= tol + ulp(got) / 2. Rows that attend a few keys,
scaled by the dropout's 1/(1 - p), have outputs of magnitude 2 to 5, where that rounding alone
is 0.0078 to 0.0156."""
import numpy as np
import pytest
import torch

import oracle
import sdpa_inputs as si
from parity import assert_matches, f64

pytestmark = pytest.mark.gpu

sdpa = pytest.importorskip("head_scaled_dot_sdpa_b200")
DEV = "cuda"
NAMES = {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}
TOL = {torch.float32: 1e-5, torch.float16: 1e-2, torch.bfloat16: 1e-2}


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


def kernel_for(q, k, v, generic=False):
    """No bias or mask: bf16/fp16 with head sizes 64 or 128 take the tcgen05 kernel when kv_len is
    a multiple of 8, else the mma.sync tiles; everything else the SIMT kernel."""
    tiles = q.dtype in (torch.bfloat16, torch.float16) and q.shape[-1] == v.shape[-1] in (64, 128)
    if generic or not tiles:
        return "weights_simt"
    return "weights_tcgen05" if k.shape[1] % 8 == 0 else "weights_mma"


SHAPES = [
    # B, Lq, Lk, H, Hkv, D, Dv
    (2, 37, 45, 4, 2, 64, 64),
    (1, 130, 200, 2, 1, 128, 128),
    (2, 64, 33, 3, 3, 40, 24),
    (2, 150, 264, 8, 2, 64, 64),
    (1, 300, 384, 4, 4, 128, 128),
    (1, 390, 136, 4, 2, 128, 128),  # more queries than keys, an odd number of query tiles
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True, "bottom_right"])
@pytest.mark.parametrize("drop_p", [0.0, 0.25])
def test_weights_shapes(dtype, shape, causal, drop_p):
    B, Lq, Lk, H, Hkv, D, Dv = shape
    q, k, v = _inputs(Lq + Lk + D, B, Lq, Lk, H, Hkv, D, Dv, dtype)
    check(q, k, v, f"{shape} causal={causal} p={drop_p}", kernel=kernel_for(q, k, v), is_causal=causal,
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


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_weights_tcgen05_lengths_and_empty_rows(dtype):
    """The tcgen05 path with per-batch offsets and lengths: a sequence with no key (NaN weights
    and output), rows before the first key (NaN), padding rows (zeros), causal bounds inside a
    tile and whole tiles past them (written by the fill kernel)."""
    q, k, v = _inputs(13, 3, 200, 264, 4, 2, 128, 128, dtype)
    check(q, k, v, "tcgen05 lengths", kernel="weights_tcgen05", is_causal=True, q_offset=[20, -5, 0],
          q_lengths=[200, 131, 12], kv_lengths=[264, 140, 0], drop_p=0.1, seed=5)
    check(q, k, v, "tcgen05 bottom right", kernel="weights_tcgen05", is_causal="bottom_right",
          q_lengths=[200, 131, 12], kv_lengths=[264, 140, 8], drop_p=0.3, seed=6)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_weights_tcgen05_scalar_offset_fill(dtype):
    """Causal with a scalar q_offset >= 0 (every row sees key 0): the statistics pass writes the
    zero weights past the causal bounds (query tile t writes those of tile nqt - 1 - t; three
    query tiles, so the middle one is its own mirror), and the last key tile holds 8 keys."""
    q, k, v = _inputs(21, 2, 300, 520, 4, 2, 128, 128, dtype)
    check(q, k, v, "tcgen05 scalar offset", kernel="weights_tcgen05", is_causal=True, q_offset=40, drop_p=0.1,
          seed=9)
    check(q, k, v, "tcgen05 scalar offset, p = 0", kernel="weights_tcgen05", is_causal=True, q_offset=200)
    # padding rows (q_lengths) with the statistics pass's fill: zeros, not NaN, past q_len
    check(q, k, v, "tcgen05 q_lengths, top left", kernel="weights_tcgen05", is_causal=True, q_lengths=[300, 77],
          drop_p=0.1, seed=10)
    check(q, k, v, "tcgen05 q_lengths, bottom right", kernel="weights_tcgen05", is_causal="bottom_right",
          q_lengths=[131, 300], drop_p=0.2, seed=12)


def test_weights_causal_gqa_workload_rows():
    """The bench's with-weights workload (causal GQA prefill shape, p = 0.1): every output row and
    the weights of a few whole (batch, head) planes against the oracle."""
    w = si.CAUSAL_GQA_PREFILL
    q, k, v = si.qkv(w)
    out, wts = sdpa.sdpa_forward_with_weights(q.to(DEV), k.to(DEV), v.to(DEV), is_causal=True, drop_p=0.1, seed=1)
    assert sdpa.last_kernel() == "weights_tcgen05"
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    out, wts = out.cpu(), wts.cpu()
    g = w.nheads // w.nkvheads
    for b, h in [(0, 0), (1, 13), (3, 31)]:
        want_o, want_w = oracle.sdpa_forward_with_weights(
            f64(q[b:b + 1, :, h:h + 1]), f64(k[b:b + 1, :, h // g:h // g + 1]), f64(v[b:b + 1, :, h // g:h // g + 1]),
            is_causal=True, drop_p=0.0)
        # the dropout draw depends on the weight's position in the whole array: compare the
        # undropped weights where the GPU kept them, and the kept fraction
        got_w = f64(wts[b, h])
        kept = got_w != 0
        tri = np.tril(np.ones((w.q_len, w.kv_len), dtype=bool))
        assert not kept[~tri].any()
        assert abs(kept[tri].mean() - (1 - 6554 / 65536)) < 0.002
        np.testing.assert_allclose(got_w[kept], want_w[0, 0][kept] / 0.9, atol=1e-2 / 2, rtol=2 ** -8)


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
