"""GPU parity at the full sizes of the workloads, in the launch configuration bench.py times,
checked on every output row against the float64 oracle (which takes the whole causal GQA
prefill in seconds on the host cores, and the others head by head or sequence by sequence)."""
import numpy as np
import pytest
import torch

import oracle
import sdpa_inputs as si
from parity import assert_matches, f64

pytestmark = pytest.mark.gpu

sdpa = pytest.importorskip("head_scaled_dot_sdpa_b200")
DEV = "cuda"


def test_causal_gqa_prefill_full_size():
    w = si.CAUSAL_GQA_PREFILL
    q, k, v = si.qkv(w)
    out = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV), is_causal=True)
    assert sdpa.last_kernel() == "prefill_tcgen05"
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    out = out.cpu()
    want = oracle.sdpa_forward(f64(q), f64(k), f64(v), is_causal=True)  # every (batch, head, row)
    assert_matches(out, want, 1e-2, "causal GQA prefill, all rows")


def test_kv_cache_decode_full_size():
    w = si.KV_CACHE_DECODE
    d = si.decode_inputs(w)
    kc, vc = d["k_cache"].to(DEV), d["v_cache"].to(DEV)
    out = sdpa.sdpa_decode_with_cache(d["q"].to(DEV), d["k_new"].to(DEV), d["v_new"].to(DEV), kc, vc,
                                      d["index"].to(DEV))
    assert sdpa.last_kernel() == "decode_splitkv"
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    out = out.cpu()
    idx = d["index"].numpy()
    for b in range(w.batch):  # every sequence
        want, kc_o, vc_o = oracle.sdpa_decode_with_cache(
            f64(d["q"][b:b + 1]), f64(d["k_new"][b:b + 1]), f64(d["v_new"][b:b + 1]),
            f64(d["k_cache"][b:b + 1]), f64(d["v_cache"][b:b + 1]), idx[b:b + 1])
        assert_matches(out[b:b + 1], want, 1e-2, f"decode b={b} (kv_len {idx[b] + 1})")
        n = idx[b] + 1
        np.testing.assert_array_equal(f64(kc[b:b + 1, :n]), kc_o[:, :n])
        np.testing.assert_array_equal(f64(vc[b:b + 1, :n]), vc_o[:, :n])


def test_alibi_t5_bias_full_size():
    w = si.ALIBI_T5_BIAS
    q, k, v = si.qkv(w)
    bias = si.alibi_t5_bias(w)
    out = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV), bias.to(DEV), is_causal=True)
    assert sdpa.last_kernel() == "prefill_tcgen05"
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    out = out.cpu()
    for h in range(w.nheads):  # every head, both batch elements at once
        want = oracle.sdpa_forward(f64(q[:, :, h:h + 1]), f64(k[:, :, h:h + 1]), f64(v[:, :, h:h + 1]),
                                   bias=f64(bias[h])[None, None], is_causal=True)
        assert_matches(out[:, :, h:h + 1], want, 1e-2, f"bias h={h}")


def test_block_sparse_full_size():
    w = si.BLOCK_SPARSE
    cls = si.block_classes(w)
    mask = si.mask_device(w, cls, DEV)
    info = sdpa.build_block_mask_info(mask)
    q, k, v = si.qkv(w)
    out = sdpa.sdpa_forward(q.to(DEV), k.to(DEV), v.to(DEV), block_info=info)
    assert sdpa.last_kernel() == "prefill_tcgen05"
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    out = out.cpu()
    arrays = {name: t.cpu().numpy() for name, t in info.arrays().items()}
    rng = np.random.Generator(np.random.PCG64(55))
    for h in range(w.nheads):  # every head and row
        mh = mask[h].cpu().numpy()
        # the device-built mask is the recipe's mask (rows rebuilt on the host from the recipe)
        rows = np.sort(rng.choice(w.q_len, size=8, replace=False))
        np.testing.assert_array_equal(mh[rows], si.mask_rows(w, cls, h, rows))
        want = oracle.sdpa_forward(f64(q[:, :, h:h + 1]), f64(k[:, :, h:h + 1]), f64(v[:, :, h:h + 1]),
                                   mask=mh[None, None])
        assert_matches(out[:, :, h:h + 1], want, 1e-2, f"block-sparse h={h}")
        # block classification of one block row, bit-exact against the oracle's
        qb = int(rows[0]) // 128
        ref = oracle.block_mask_info(mh[None, qb * 128:qb * 128 + 128], 128, 128)
        np.testing.assert_array_equal(arrays["cls"][h, qb], ref["cls"][0, 0])
        n = int(ref["count"][0, 0])
        assert arrays["count"][h, qb] == n
        np.testing.assert_array_equal(arrays["list"][h, qb, :n].view(np.uint32), ref["list"][0, 0, :n])
        for kb in np.nonzero(ref["cls"][0, 0] == 1)[0]:
            np.testing.assert_array_equal(arrays["bits"][h, qb, kb].view(np.uint32), ref["bits"][0, 0, kb])
