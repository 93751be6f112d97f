"""GPU parity of packed sequences (keywords q_segments, kv_segments and maxlen of
NNlib.scaled_dot_product_attention, paragraph "Packed sequences") against the CPU oracle,
through the C ABI: the tcgen05 kernel for bf16/f16 at head_dim 64/128, the SIMT kernel for
fp32 and other head sizes."""
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


def _packed(seed, qs, ks, H, Hkv, D, dtype):
    rng = np.random.Generator(np.random.PCG64(seed))
    n = NAMES[dtype]
    return (si.normal(rng, (sum(qs), H, D), n), si.normal(rng, (sum(ks), Hkv, D), n),
            si.normal(rng, (sum(ks), Hkv, D), n))


def run(q, k, v, qs, ks=None, kernel="prefill_tcgen05", **kw):
    out = sdpa.sdpa_forward_packed(q.to(DEV), k.to(DEV), v.to(DEV), qs, ks, **kw)
    assert sdpa.last_kernel() == kernel
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    return out


# query segments, key/value segments (None: the same): one row, a tile less one, exactly a
# tile, a tile and one, several tiles with a ragged tail, an empty segment
SEGMENTS = [
    ([1, 127, 128, 129, 300, 0, 45], None),
    ([100, 0, 257, 33], [64, 5, 300, 1]),
    ([513], None),
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("segs", SEGMENTS, ids=lambda s: f"{len(s[0])}seg")
@pytest.mark.parametrize("causal", [False, True, "bottom_right"])
def test_packed_tcgen05(dtype, D, segs, causal):
    qs, ks = segs
    kv = ks or qs
    q, k, v = _packed(sum(qs) + 3 * D, qs, kv, 8, 2, D, dtype)
    out = run(q, k, v, qs, ks, is_causal=causal)
    want = oracle.sdpa_forward_packed(f64(q), f64(k), f64(v), qs, ks, is_causal=causal)
    assert_matches(out, want, 1e-2, f"packed {qs}/{kv} causal={causal}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_packed_offsets_and_lengths(dtype):
    """Per-segment q_offset, q_lengths and kv_lengths (rows past q_lengths are zero, a segment
    whose queries see no key is NaN)."""
    qs, ks = [130, 7, 260, 64], [200, 9, 260, 0]
    q, k, v = _packed(11, qs, ks, 4, 4, 128, dtype)
    kw = dict(is_causal=True, q_offset=[70, 2, 0, 0], q_lengths=[129, 7, 200, 64], kv_lengths=[150, 9, 259, 0])
    out = run(q, k, v, qs, ks, **kw)
    want = oracle.sdpa_forward_packed(f64(q), f64(k), f64(v), qs, ks, **kw)
    assert_matches(out, want, 1e-2, "packed offsets/lengths")
    kw = dict(is_causal="bottom_right", q_lengths=[100, 3, 260, 10], kv_lengths=[200, 5, 100, 0])
    out = run(q, k, v, qs, ks, **kw)
    want = oracle.sdpa_forward_packed(f64(q), f64(k), f64(v), qs, ks, **kw)
    assert_matches(out, want, 1e-2, "packed bottom-right lengths")


def test_packed_printed_example_fp32():
    """The page's example: x of size (16, 8, 20), is_causal, q_segments [5, 12, 3] (SIMT kernel)."""
    x = _packed(12, [20], [20], 8, 8, 16, torch.float32)[0]
    out = run(x, x, x, [5, 12, 3], kernel="generic_simt", is_causal=True)
    assert out.shape == x.shape
    want = oracle.sdpa_forward_packed(f64(x), f64(x), f64(x), [5, 12, 3], is_causal=True)
    assert_matches(out, want, 1e-5, "printed packed example")


@pytest.mark.parametrize("D", [128, 80])
def test_packed_fp32_and_generic(D):
    qs, ks = [33, 0, 140, 2], [40, 3, 140, 1]
    q, k, v = _packed(13 + D, qs, ks, 6, 3, D, torch.float32)
    out = run(q, k, v, qs, ks, kernel="generic_simt", is_causal=True, q_offset=[7, 0, 0, 0])
    want = oracle.sdpa_forward_packed(f64(q), f64(k), f64(v), qs, ks, is_causal=True, q_offset=[7, 0, 0, 0])
    assert_matches(out, want, 1e-5, f"packed fp32 D={D}")
    qb, kb, vb = (t.to(torch.bfloat16) for t in (q, k, v))
    out = run(qb, kb, vb, qs, ks, kernel="generic_simt", generic=True, is_causal=True)
    want = oracle.sdpa_forward_packed(f64(qb), f64(kb), f64(vb), qs, ks, is_causal=True)
    assert_matches(out, want, 1e-2, f"packed bf16 forced SIMT D={D}")


def test_packed_equals_padded_batch_bitwise():
    """Equal segments that start on tile boundaries are a padded batch: the same tiles are
    loaded and reduced in the same order, so the outputs agree bit for bit."""
    B, L, H, Hkv, D = 3, 384, 8, 2, 128
    q, k, v = _packed(14, [B * L], [B * L], H, Hkv, D, torch.bfloat16)
    packed = run(q, k, v, [L] * B, is_causal=True)
    padded = sdpa.sdpa_forward(q.view(B, L, H, D).to(DEV), k.view(B, L, Hkv, D).to(DEV),
                               v.view(B, L, Hkv, D).to(DEV), is_causal=True)
    assert torch.equal(packed, padded.view(B * L, H, D))


def test_packed_device_segments_and_maxlen():
    """Lengths given as a device tensor, with and without maxlen (without it the binding reads
    them back to find it)."""
    qs = [5, 200, 0, 131]
    q, k, v = _packed(15, qs, qs, 4, 2, 64, torch.bfloat16)
    seg = torch.tensor(qs, dtype=torch.int32, device=DEV)
    want = oracle.sdpa_forward_packed(f64(q), f64(k), f64(v), qs, is_causal=True)
    for maxlen in (200, 1000, None):
        out = run(q, k, v, seg, is_causal=True, maxlen=maxlen)
        assert_matches(out, want, 1e-2, f"device segments maxlen={maxlen}")


def test_packed_docs_workload_sampled():
    """The benchmark's packed workload at its full size (30 documents packed into 65536
    positions, 32 query / 8 key-value heads, head_dim 128, causal), launched as the benchmark
    launches it. Sampled query rows of four documents are checked against the oracle run on
    each document alone (its keys up to the sampled row)."""
    w = si.PACKED_DOCS
    segs = si.packed_segments(w)
    q, k, v = si.packed_qkv(w)
    seg = torch.tensor(segs, dtype=torch.int32, device=DEV)
    out = run(q, k, v, seg, is_causal=True, maxlen=max(segs)).cpu()
    starts = np.cumsum([0] + segs)
    rng = np.random.Generator(np.random.PCG64(16))
    for s in (0, 7, len(segs) // 2, len(segs) - 1):
        a, n = int(starts[s]), segs[s]
        rows = sorted({0, n - 1, *(int(x) for x in rng.integers(0, n, size=6))})
        for i in rows:
            want = oracle.sdpa_forward_packed(f64(q[a + i:a + i + 1]), f64(k[a:a + i + 1]), f64(v[a:a + i + 1]),
                                              [1], [i + 1], is_causal=True, q_offset=[i])
            assert_matches(out[a + i:a + i + 1], want, 1e-2, f"document {s} row {i}")


def test_packed_device_checks():
    """Lengths the host never reads are checked on the device: a segment above maxlen, or
    lengths that do not add up to the array rows, set SDPA_ERR_DEVICE_CHECK; every access stays
    inside the arrays."""
    q, k, v = _packed(18, [300], [300], 2, 2, 128, torch.bfloat16)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    for segs, maxlen in (([100, 200], 150), ([100, 150], 200), ([100, 250], 250), ([-5, 305], 305)):
        seg = torch.tensor(segs, dtype=torch.int32, device=DEV)
        sdpa.sdpa_forward_packed(qd, kd, vd, seg, maxlen=maxlen)
        assert sdpa.read_device_status() == sdpa.SDPA_ERR_DEVICE_CHECK, (segs, maxlen)
    # valid lengths afterwards give the right answer again
    out = run(q, k, v, [100, 200])
    assert_matches(out, oracle.sdpa_forward_packed(f64(q), f64(k), f64(v), [100, 200]), 1e-2, "after checks")


def test_packed_host_errors():
    q, k, v = (t.to(DEV) for t in _packed(19, [64], [64], 2, 2, 64, torch.bfloat16))
    with pytest.raises(ValueError):
        sdpa.sdpa_forward_packed(q, k, v, [32, 32], [32, 32, 0])
    with pytest.raises(sdpa.SdpaError):
        sdpa.sdpa_forward_packed(q, k, v, [], maxlen=0)  # no segments for 64 rows
