"""GPU parity of the SIMT attention kernel, the split-KV decode, the cache update and the block
classification against the CPU oracle, through the C ABI (Python binding)."""
import numpy as np
import pytest
import torch

import oracle
import sdpa_inputs as si
from parity import TOL, assert_matches, f64

pytestmark = pytest.mark.gpu

sdpa = pytest.importorskip("head_scaled_dot_sdpa_b200")
DEV = "cuda"


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _qkv(seed, B, Lq, Lk, H, Hkv, D, Dv, dtype):
    rng = _rng(seed)
    mk = lambda s: si.normal(rng, s, {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}[dtype])
    return mk((B, Lq, H, D)), mk((B, Lk, Hkv, D)), mk((B, Lk, Hkv, Dv))


def test_tiny_fp32_workload():
    w = si.TINY_FP32
    q, k, v = si.qkv(w)
    out = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV))
    assert sdpa.last_kernel() == "generic_simt"
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v))
    assert out.shape == (1, 8, 2, 16)
    assert_matches(out, want, 1e-5, "tiny fp32")
    assert sdpa.read_device_status() == sdpa.SDPA_OK


CASES = [
    # name, kwargs for shapes, call kwargs builder
    ("plain_gqa", dict(B=2, Lq=37, Lk=45, H=8, Hkv=2, D=64, Dv=64), {}),
    ("causal_top_left_offsets", dict(B=3, Lq=33, Lk=50, H=4, Hkv=4, D=32, Dv=48),
     dict(is_causal=True, q_offset=[0, 5, 17])),
    ("bottom_right_lengths", dict(B=3, Lq=20, Lk=70, H=4, Hkv=1, D=64, Dv=64),
     dict(is_causal="bottom_right", q_lengths=[20, 7, 1], kv_lengths=[70, 33, 9])),
    ("negative_offset_nan_rows", dict(B=1, Lq=10, Lk=10, H=2, Hkv=2, D=16, Dv=16),
     dict(is_causal=True, q_offset=-3)),
    ("scale_and_dv", dict(B=1, Lq=9, Lk=65, H=2, Hkv=1, D=80, Dv=24), dict(scale=0.37)),
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("name,shape,kw", CASES, ids=[c[0] for c in CASES])
def test_generic_kernel_semantics(name, shape, kw, dtype):
    q, k, v = _qkv(sum(map(ord, name)), shape["B"], shape["Lq"], shape["Lk"], shape["H"], shape["Hkv"],
                   shape["D"], shape["Dv"], dtype)
    out = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV), generic=True, **kw)
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v), **kw)
    assert_matches(out, want, TOL[dtype], name)
    assert sdpa.read_device_status() == sdpa.SDPA_OK


@pytest.mark.parametrize("bias_dtype", [torch.float32, torch.bfloat16])
def test_generic_bias_and_mask(bias_dtype):
    rng = _rng(7)
    B, Lq, Lk, H, Hkv, D = 2, 19, 41, 4, 2, 64
    q, k, v = _qkv(8, B, Lq, Lk, H, Hkv, D, D, torch.bfloat16)
    bias = torch.from_numpy(rng.standard_normal((1, H, Lq, Lk)).astype(np.float32)).to(bias_dtype)
    mask = torch.from_numpy(rng.random((B, 1, Lq, Lk)) < 0.6)
    mask[..., 3] = True
    out = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV), bias.to(DEV), mask=mask.to(DEV),
                            is_causal=True, q_offset=10, kv_lengths=[41, 30], generic=True)
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v), bias=f64(bias), mask=mask.numpy(), is_causal=True,
                               q_offset=10, kv_lengths=[41, 30])
    assert_matches(out, want, 1e-2, "bias+mask")


def test_degenerate_sizes():
    q, k, v = _qkv(9, 2, 0, 5, 2, 2, 16, 16, torch.bfloat16)
    out = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV))
    assert out.shape == (2, 0, 2, 16)
    q, k, v = _qkv(9, 2, 4, 5, 2, 2, 16, 16, torch.bfloat16)
    out = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV), kv_lengths=[0, 5])
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v), kv_lengths=[0, 5])
    assert_matches(out, want, 1e-2, "kv_length 0 -> NaN")
    assert torch.isnan(out[0]).all()


# ---- KV-cache decode --------------------------------------------------------------------------

def _decode_case(B, cap, H, Hkv, D, n_new, dtype, seed, lo=1):
    rng = _rng(seed)
    name = {torch.float16: "f16", torch.bfloat16: "bf16", torch.float32: "f32"}[dtype]
    kv_lengths = rng.integers(max(lo, n_new), cap, size=B, endpoint=True)
    idx = (kv_lengths - n_new).astype(np.int32)
    q = si.normal(rng, (B, n_new, H, D), name)
    kn = si.normal(rng, (B, n_new, Hkv, D), name)
    vn = si.normal(rng, (B, n_new, Hkv, D), name)
    kc = si.normal(rng, (B, cap, Hkv, D), name)
    vc = si.normal(rng, (B, cap, Hkv, D), name)
    return q, kn, vn, kc, vc, idx


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("D,H,Hkv,n_new", [(128, 32, 8, 1), (128, 8, 2, 3), (64, 16, 16, 1), (128, 4, 4, 4)])
@pytest.mark.parametrize("generic", [False, True])
def test_decode_with_cache(dtype, D, H, Hkv, n_new, generic):
    B, cap = 5, 1100
    q, kn, vn, kc, vc, idx = _decode_case(B, cap, H, Hkv, D, n_new, dtype, seed=D + H + n_new)
    kc_d, vc_d = kc.to(DEV), vc.to(DEV)
    out = sdpa.sdpa_decode_with_cache(q.to(DEV), kn.to(DEV), vn.to(DEV), kc_d, vc_d,
                                      torch.from_numpy(idx), generic=generic)
    expected_kernel = "generic_simt" if generic or H // Hkv * n_new > 16 else "decode_splitkv"
    assert sdpa.last_kernel() == expected_kernel
    want, kc_o, vc_o = oracle.sdpa_decode_with_cache(f64(q), f64(kn), f64(vn), f64(kc), f64(vc), idx)
    assert_matches(out, want, 1e-2, "decode")
    np.testing.assert_array_equal(f64(kc_d), kc_o)  # the copy is exact
    np.testing.assert_array_equal(f64(vc_d), vc_o)
    assert sdpa.read_device_status() == sdpa.SDPA_OK


@pytest.mark.parametrize("generic", [False, True])
def test_decode_bad_index_nan_rows(generic):
    """A cache index out of range skips that sequence (cache untouched), writes NaN to its output
    rows and sets the status word; the other sequences match the oracle."""
    B, cap, H, Hkv, D = 4, 300, 8, 2, 128
    q, kn, vn, kc, vc, idx = _decode_case(B, cap, H, Hkv, D, 2, torch.bfloat16, seed=11)
    idx = idx.copy()
    idx[1] = cap - 1  # a 2-token write would end past the capacity
    idx[3] = -1
    kc_d, vc_d = kc.to(DEV), vc.to(DEV)
    ws = sdpa.Workspace(DEV)
    out = sdpa.sdpa_decode_with_cache(q.to(DEV), kn.to(DEV), vn.to(DEV), kc_d, vc_d, torch.from_numpy(idx),
                                      generic=generic, workspace=ws)
    assert sdpa.read_device_status(ws) == sdpa.SDPA_ERR_DEVICE_CHECK
    got = out.cpu()
    for b in (1, 3):
        assert torch.isnan(got[b].float()).all()
        np.testing.assert_array_equal(f64(kc_d[b]), f64(kc[b]))
    good = np.array([0, 2])
    want, _, _ = oracle.sdpa_decode_with_cache(f64(q[good]), f64(kn[good]), f64(vn[good]), f64(kc[good]),
                                               f64(vc[good]), idx[good])
    assert_matches(got[good], want, 1e-2, "decode next to bad indices")


def test_decode_split_boundaries():
    """Lengths at and around the split size, and a single key."""
    B, cap, H, Hkv, D = 8, 2048, 8, 2, 128
    q, kn, vn, kc, vc, _ = _decode_case(B, cap, H, Hkv, D, 1, torch.bfloat16, seed=5)
    idx = np.array([0, 15, 16, 511, 512, 1023, 1024, 2047], dtype=np.int32)
    out = sdpa.sdpa_decode_with_cache(q.to(DEV), kn.to(DEV), vn.to(DEV), kc.to(DEV), vc.to(DEV),
                                      torch.from_numpy(idx))
    want, _, _ = oracle.sdpa_decode_with_cache(f64(q), f64(kn), f64(vn), f64(kc), f64(vc), idx)
    assert_matches(out, want, 1e-2, "decode split boundaries")
    # one key: the output is that key's value exactly (after rounding)
    np.testing.assert_allclose(f64(out[0, 0]), f64(vn[0, 0]).repeat(H // Hkv, axis=0), atol=1e-2)


def test_cache_update_and_bad_index():
    B, cap, Hkv, D = 4, 64, 2, 128
    rng = _rng(3)
    kc = si.normal(rng, (B, cap, Hkv, D), "bf16")
    kn = si.normal(rng, (B, 2, Hkv, D), "bf16")
    idx = np.array([0, 62, 10, 63], dtype=np.int32)  # the last one is out of range for 2 rows
    kc_d = kc.to(DEV)
    ws = sdpa.Workspace(DEV)
    sdpa.cache_update_at_index(kc_d, None, kn.to(DEV), None, torch.from_numpy(idx), workspace=ws)
    assert sdpa.read_device_status(ws) == sdpa.SDPA_ERR_DEVICE_CHECK
    assert sdpa.read_device_status(ws) == sdpa.SDPA_OK  # cleared by the read
    want = oracle.cache_update_at_index(f64(kc[:3]), f64(kn[:3]), idx[:3])
    np.testing.assert_array_equal(f64(kc_d[:3]), want)
    np.testing.assert_array_equal(f64(kc_d[3]), f64(kc[3]))  # skipped sequence untouched


# ---- block classification ---------------------------------------------------------------------

@pytest.mark.parametrize("H,Lq,Lk,bq,bk", [(2, 300, 260, 64, 64), (3, 256, 384, 128, 128),
                                          (1, 131, 200, 128, 128), (2, 40, 96, 16, 32)])
def test_block_classification_bit_exact(H, Lq, Lk, bq, bk):
    w = si.scaled(si.BLOCK_SPARSE, nheads=H, q_len=Lq, kv_len=Lk, block=bq)
    cls = si.block_classes(w) if bq == bk else None
    mask = si.mask_device(w, cls, DEV) if cls is not None else \
        torch.from_numpy((_rng(4).random((H, Lq, Lk)) < 0.5).astype(np.uint8)).to(DEV)
    info = sdpa.build_block_mask_info(mask, bq, bk)
    got = {k: t.cpu().numpy() for k, t in info.arrays().items()}
    want = oracle.block_mask_info(mask.cpu().numpy(), bq, bk)
    np.testing.assert_array_equal(got["cls"], want["cls"])
    np.testing.assert_array_equal(got["count"], want["count"])
    for h in range(H):
        for qb in range(want["count"].shape[1]):
            n = want["count"][h, qb]
            np.testing.assert_array_equal(got["list"][h, qb, :n].view(np.uint32), want["list"][h, qb, :n])
            for kb in np.nonzero(want["cls"][h, qb] == 1)[0]:
                np.testing.assert_array_equal(got["bits"][h, qb, kb].view(np.uint32), want["bits"][h, qb, kb])


def test_forward_with_block_info_generic():
    w = si.scaled(si.BLOCK_SPARSE, nheads=2, q_len=300, kv_len=420, block=128)
    cls = si.block_classes(w)
    mask = si.mask_device(w, cls, DEV)
    info = sdpa.build_block_mask_info(mask, 128, 128)
    q, k, v = _qkv(11, 1, 300, 420, 2, 2, 128, 128, torch.bfloat16)
    out = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV), block_info=info, generic=True)
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v), mask=mask.cpu().numpy()[None])
    assert_matches(out, want, 1e-2, "block info (generic)")
