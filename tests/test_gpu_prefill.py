"""GPU parity of the tcgen05 prefill kernel against the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import sdpa_inputs as si
from parity import assert_matches, f64

pytestmark = pytest.mark.gpu

sdpa = pytest.importorskip("head_scaled_dot_sdpa_b200")
DEV = "cuda"
NAMES = {torch.float16: "f16", torch.bfloat16: "bf16"}


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _qkv(seed, B, Lq, Lk, H, Hkv, D, dtype):
    rng = _rng(seed)
    n = NAMES[dtype]
    return (si.normal(rng, (B, Lq, H, D), n), si.normal(rng, (B, Lk, Hkv, D), n),
            si.normal(rng, (B, Lk, Hkv, D), n))


def run(q, k, v, bias=None, **kw):
    out = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV), bias, **kw)
    assert sdpa.last_kernel() == "prefill_tcgen05"
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    return out


SHAPES = [
    # B, Lq, Lk, H, Hkv
    (1, 128, 128, 1, 1),
    (2, 300, 300, 4, 2),
    (1, 37, 45, 2, 1),
    (2, 256, 700, 8, 2),
    (1, 700, 256, 2, 2),
    (1, 200, 300, 6, 2),    # GQA group of 3: one unit has no second head
    (2, 640, 640, 3, 3),    # odd number of query tiles: the last unit has one tile
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True, "bottom_right"])
def test_prefill_shapes(dtype, D, shape, causal):
    B, Lq, Lk, H, Hkv = shape
    q, k, v = _qkv(Lq * 7 + Lk + D, B, Lq, Lk, H, Hkv, D, dtype)
    out = run(q, k, v, is_causal=causal)
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v), is_causal=causal)
    assert_matches(out, want, 1e-2, f"{shape} causal={causal}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_prefill_lengths_offsets(dtype):
    B, Lq, Lk, H, Hkv, D = 3, 260, 400, 4, 1, 128
    q, k, v = _qkv(21, B, Lq, Lk, H, Hkv, D, dtype)
    cases = [
        dict(is_causal=True, q_offset=[0, 100, 300]),
        dict(is_causal=True, q_offset=-50),
        dict(is_causal="bottom_right", q_lengths=[260, 129, 1], kv_lengths=[400, 200, 130]),
        dict(kv_lengths=[1, 128, 399], q_lengths=[5, 260, 200]),
        dict(is_causal=True, kv_lengths=[0, 50, 400]),
        dict(scale=0.05),
    ]
    for kw in cases:
        out = run(q, k, v, **kw)
        want = oracle.sdpa_forward(f64(q), f64(k), f64(v), **kw)
        assert_matches(out, want, 1e-2, str(kw))


@pytest.mark.parametrize("bias_dtype", [torch.float16, torch.float32])
def test_prefill_bias_and_mask(bias_dtype):
    # rows of 336 keys are 16-byte aligned for both bias and mask: the tcgen05 kernel takes them
    B, Lq, Lk, H, Hkv, D = 2, 200, 336, 4, 2, 64
    rng = _rng(5)
    q, k, v = _qkv(6, B, Lq, Lk, H, Hkv, D, torch.float16)
    bias = torch.from_numpy((rng.standard_normal((H, Lq, Lk)) * 2).astype(np.float32)).to(bias_dtype)
    mask = torch.from_numpy(rng.random((B, 1, Lq, Lk)) < 0.7)
    mask[..., 0] = True
    kw = dict(is_causal=True, q_offset=40)
    out = run(q, k, v, bias.to(DEV), mask=mask.to(DEV), **kw)
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v), bias=f64(bias), mask=mask.numpy(), **kw)
    assert_matches(out, want, 1e-2, "bias+mask")


BIAS_LAYOUTS = {
    # shape of the bias tensor, broadcast to (B, H, Lq, Lk)
    "bhqk": lambda B, H, Lq, Lk: (B, H, Lq, Lk),
    "qk": lambda B, H, Lq, Lk: (Lq, Lk),          # shared by every batch element and head
    "b1qk": lambda B, H, Lq, Lk: (B, 1, Lq, Lk),  # shared by the heads
    "hk": lambda B, H, Lq, Lk: (H, 1, Lk),        # one row per head, shared by the queries
}


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layout", list(BIAS_LAYOUTS))
@pytest.mark.parametrize("causal", [False, True])
def test_prefill_bias_layouts(D, layout, causal):
    # 272 keys: 16-byte aligned rows; 300 queries: three query tiles (one unit with one tile)
    B, Lq, Lk, H, Hkv = 2, 300, 272, 4, 2
    rng = _rng(11 + D)
    q, k, v = _qkv(12 + D, B, Lq, Lk, H, Hkv, D, torch.bfloat16)
    # unit-variance bias (ALiBi / T5 magnitudes): a near one-hot softmax would put outputs of
    # |v| ~ 3 on the bf16 grid, whose half-spacing there (0.0078) alone nearly fills 1e-2
    bias = torch.from_numpy(rng.standard_normal(BIAS_LAYOUTS[layout](B, H, Lq, Lk)).astype(np.float32))
    bias = bias.to(torch.bfloat16)
    out = run(q, k, v, bias.to(DEV), is_causal=causal)
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v), bias=f64(bias), is_causal=causal)
    assert_matches(out, want, 1e-2, f"bias {layout} D={D}")


@pytest.mark.parametrize("D", [64, 128])
def test_prefill_bias_with_block_info(D):
    # a 16-bit bias (through shared-memory tiles at head_dim 64) together with the partial-block
    # bits of a block-sparse mask
    w = si.scaled(si.BLOCK_SPARSE, nheads=4, q_len=640, kv_len=768, block=128)
    cls = si.block_classes(w)
    mask = si.mask_device(w, cls, DEV)
    info = sdpa.build_block_mask_info(mask, 128, 128)
    rng = _rng(21 + D)
    q, k, v = _qkv(22 + D, 1, 640, 768, 4, 4, D, torch.float16)
    bias = torch.from_numpy(rng.standard_normal((4, 640, 768)).astype(np.float32)).to(torch.float16)
    out = run(q, k, v, bias.to(DEV), block_info=info)
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v), bias=f64(bias), mask=mask.cpu().numpy()[None])
    assert_matches(out, want, 1e-2, f"bias + block info D={D}")


def test_prefill_block_info():
    w = si.scaled(si.BLOCK_SPARSE, nheads=4, q_len=600, kv_len=900, block=128)
    cls = si.block_classes(w)
    mask = si.mask_device(w, cls, DEV)
    info = sdpa.build_block_mask_info(mask, 128, 128)
    q, k, v = _qkv(7, 1, 600, 900, 4, 4, 128, torch.bfloat16)
    out = run(q, k, v, block_info=info)
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v), mask=mask.cpu().numpy()[None])
    assert_matches(out, want, 1e-2, "block info")
    # the dense mask itself (900 keys per row: not 16-byte aligned, so the SIMT kernel) agrees
    out2 = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV), mask=mask)
    assert_matches(out2, want, 1e-2, "dense mask")
    # an aligned dense mask goes through the tcgen05 kernel's dense-mask variant
    out3 = run(q[:, :, :, :], k[:, :896], v[:, :896], mask=mask[:, :, :896].contiguous())
    want3 = oracle.sdpa_forward(f64(q), f64(k[:, :896]), f64(v[:, :896]), mask=mask[:, :, :896].cpu().numpy()[None])
    assert_matches(out3, want3, 1e-2, "dense mask (tcgen05)")


def test_prefill_empty_rows_and_all_masked_blocks():
    B, Lq, Lk, H, D = 1, 256, 256, 2, 128
    q, k, v = _qkv(8, B, Lq, Lk, H, H, D, torch.bfloat16)
    mask = torch.ones((1, H, Lq, Lk), dtype=torch.bool)
    mask[0, 0, 5, :] = False           # one empty row
    mask[0, 1, 128:, :128] = False     # a whole empty block
    out = run(q, k, v, mask=mask.to(DEV))
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v), mask=mask.numpy())
    assert_matches(out, want, 1e-2, "empty rows")
    assert torch.isnan(out[0, 5, 0]).all()


def test_unaligned_mask_takes_the_simt_kernel():
    """A mask whose rows are not 16-byte aligned is not read by the tcgen05 kernel; the SIMT
    kernel computes the call instead, with the same result."""
    B, Lq, Lk, H, D = 1, 100, 333, 2, 64
    rng = _rng(9)
    q, k, v = _qkv(10, B, Lq, Lk, H, H, D, torch.float16)
    mask = torch.from_numpy(rng.random((B, H, Lq, Lk)) < 0.6)
    mask[..., 0] = True
    out = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV), mask=mask.to(DEV))
    assert sdpa.last_kernel() == "generic_simt"
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v), mask=mask.numpy())
    assert_matches(out, want, 1e-2, "unaligned mask")


def test_bounded_wait_reports_timeout_and_context_survives():
    """Every mbarrier wait of the tcgen05 kernel is bounded. The self-test flag makes the TMA
    producer wait on a phase nothing completes (with 1 ms bounds): the call must end with
    SDPA_ERR_TIMEOUT in the status word, and the next call must run normally."""
    q, k, v = _qkv(12, 1, 256, 256, 2, 2, 128, torch.bfloat16)
    ws = sdpa.Workspace(DEV)
    sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV), workspace=ws, flags=sdpa.SDPA_FLAG_SELFTEST_STALL)
    assert sdpa.last_kernel() == "prefill_tcgen05"
    assert sdpa.read_device_status(ws) == sdpa.SDPA_ERR_TIMEOUT
    out = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV), workspace=ws)
    assert sdpa.read_device_status(ws) == sdpa.SDPA_OK
    assert_matches(out, oracle.sdpa_forward(f64(q), f64(k), f64(v)), 1e-2, "after the timeout")
