"""The seeded input recipes: reproducible, with the stated structure."""
import numpy as np
import torch

import sdpa_inputs as si


def test_mask_generators_agree_and_keep_a_key_per_row():
    w = si.scaled(si.BLOCK_SPARSE, nheads=2, q_len=300, kv_len=260, block=64)
    cls = si.block_classes(w)
    dev = si.mask_device(w, cls, "cpu").numpy()
    for h in range(2):
        rows = np.arange(w.q_len)
        np.testing.assert_array_equal(si.mask_rows(w, cls, h, rows), dev[h])
    assert dev.sum(axis=-1).min() >= 1
    assert (dev[:, np.arange(260), np.arange(260)] == 1).all()
    # empty/full blocks away from the diagonal are exactly empty/full
    for h in range(2):
        for qb in range(cls.shape[1]):
            for kb in range(cls.shape[2]):
                if qb == kb:
                    continue
                blk = dev[h, qb * 64:(qb + 1) * 64, kb * 64:(kb + 1) * 64]
                if cls[h, qb, kb] == 0:
                    assert blk.sum() == 0
                elif cls[h, qb, kb] == 2:
                    assert blk.all()


def test_block_class_frequencies():
    cls = si.block_classes(si.BLOCK_SPARSE)
    assert cls.shape == (16, 128, 128)
    f = np.bincount(cls.ravel(), minlength=3) / cls.size
    assert abs(f[0] - 0.5) < 0.01 and abs(f[1] - 0.2) < 0.01 and abs(f[2] - 0.3) < 0.01


def test_decode_inputs_lengths_and_index():
    w = si.scaled(si.KV_CACHE_DECODE, batch=8, capacity=64, kv_len=64, kv_len_min=5, kv_len_max=64)
    d = si.decode_inputs(w)
    kl = d["kv_lengths"].numpy()
    assert kl.min() >= 5 and kl.max() <= 64
    np.testing.assert_array_equal(d["index"].numpy(), kl - 1)
    assert d["k_cache"].dtype == torch.bfloat16 and d["k_cache"].shape == (8, 64, 8, 128)


def test_alibi_bias_structure():
    w = si.scaled(si.ALIBI_T5_BIAS, nheads=4, q_len=16, kv_len=16, bias_noise_std=0.0)
    b = si.alibi_t5_bias(w).float().numpy()
    # head 1 of 4: slope 2^(-2); entry (i, j) = slope * (j - i)
    assert b[0, 3, 7] == 0.25 * 4 and b[0, 7, 3] == -0.25 * 4
    assert b[3, 0, 5] == 2.0 ** -8 * 5


def test_reproducible():
    a = si.qkv(si.TINY_FP32)
    b = si.qkv(si.TINY_FP32)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_packed_documents_recipe():
    """Lengths in [seg_min, seg_max] (the last one cut to fit) adding up to the packed total;
    the same seed gives the same documents."""
    w = si.PACKED_DOCS
    segs = si.packed_segments(w)
    assert sum(segs) == w.q_len == w.kv_len
    assert all(w.seg_min <= n <= w.seg_max for n in segs[:-1]) and 1 <= segs[-1] <= w.seg_max
    assert segs == si.packed_segments(w) and len(segs) == 30
    q, k, v = si.packed_qkv(si.scaled(w, q_len=100, kv_len=100))
    assert q.shape == (100, 32, 128) and k.shape == v.shape == (100, 8, 128)


def test_causal_pair_count():
    """bench.causal_pairs (the flop count of every causal workload) against counting."""
    import bench
    for lq, lk, off in ((7, 7, 0), (5, 9, 4), (9, 5, -2), (1, 8192, 8191), (64, 64, -70)):
        i = np.arange(lq)[:, None]
        j = np.arange(lk)[None, :]
        assert bench.causal_pairs(lq, lk, off) == int((j <= off + i).sum())
