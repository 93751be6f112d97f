"""Pins of the CPU oracle to facts outside itself.

Every pin checks the oracle against something the page or mathematics fixes: a closed form,
an equivalence the entry states, PyTorch's float64 CPU routine on the special cases it can
express, or brute-force counting. Each takes the oracle library handle, so that the mutant
tests can run the same pins against deliberately broken builds of the oracle.

Passages cited are from the Flux.jl page "Neural Network primitives from NNlib.jl", entry
NNlib.scaled_dot_product_attention, unless stated otherwise.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
PINS = []


def pin(fn):
    PINS.append(fn)
    return fn


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _qkv(rng, B, Lq, Lk, H, Hkv, D, Dv=None):
    Dv = Dv or D
    q = rng.standard_normal((B, Lq, H, D))
    k = rng.standard_normal((B, Lk, Hkv, D))
    v = rng.standard_normal((B, Lk, Hkv, Dv))
    return q, k, v


def _torch_sdpa(q, k, v, **kw):
    """PyTorch's float64 CPU scaled_dot_product_attention in our layout. PyTorch's layout is
    (batch, nheads, seq, dim), so the seq and head axes are swapped on the way in and out
    (the entry's layout paragraph warns of exactly this permutation)."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).permute(0, 2, 1, 3)
    am = kw.pop("attn_mask", None)
    if am is not None:
        am = torch.from_numpy(np.ascontiguousarray(am))
    out = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=am, **kw)
    return out.permute(0, 2, 1, 3).numpy()


def _close(a, b, tol=1e-12):
    np.testing.assert_allclose(a, b, rtol=0, atol=tol)


# ---- library routine on the special cases it expresses ------------------------------------

@pin
def torch_plain_unequal_lengths_dv(lib):
    """First paragraph: softmax(scale·qᵀk)·v with the default scale 1/√qk_head_dim, and a
    value head size different from the query's (Returns: (v_head_dim, nheads, q_len, ...))."""
    q, k, v = _qkv(_rng(11), 2, 5, 7, 3, 3, 8, 6)
    _close(oracle.sdpa_forward(q, k, v, lib=lib), _torch_sdpa(q, k, v))


@pin
def torch_causal_top_left(lib):
    """Argument is_causal=true: query i attends keys j ≤ i (q_offset 0), for equal and for
    unequal lengths; PyTorch's is_causal is the same top-left alignment."""
    for (Lq, Lk) in ((6, 6), (4, 9), (9, 4)):
        q, k, v = _qkv(_rng(12 + Lq), 2, Lq, Lk, 2, 2, 8)
        _close(oracle.sdpa_forward(q, k, v, is_causal=True, lib=lib),
               _torch_sdpa(q, k, v, is_causal=True))


@pin
def torch_gqa(lib):
    """GQA paragraph: fewer key/value heads shared across query heads; PyTorch's enable_gqa
    repeats each key/value head over a contiguous group of query heads."""
    q, k, v = _qkv(_rng(13), 2, 5, 6, 8, 2, 8)
    _close(oracle.sdpa_forward(q, k, v, lib=lib), _torch_sdpa(q, k, v, enable_gqa=True))


@pin
def torch_bool_mask_broadcast(lib):
    """Argument mask: a boolean array broadcastable to (kv_len, q_len, nheads, batch), i.e.
    row-major (batch, nheads, q_len, kv_len); false entries are not attended."""
    rng = _rng(14)
    q, k, v = _qkv(rng, 2, 5, 7, 3, 3, 8)
    mask = rng.random((1, 3, 5, 7)) < 0.6  # broadcast over batch
    mask[..., 0] = True  # keep one key per row
    _close(oracle.sdpa_forward(q, k, v, mask=mask, lib=lib),
           _torch_sdpa(q, k, v, attn_mask=np.broadcast_to(mask, (2, 3, 5, 7)).copy()))


@pin
def torch_float_bias_and_scale(lib):
    """Arguments bias and scale: the bias is added to the scaled logits before the softmax."""
    rng = _rng(15)
    q, k, v = _qkv(rng, 2, 4, 6, 2, 2, 8)
    bias = rng.standard_normal((2, 1, 4, 6))  # broadcast over heads
    _close(oracle.sdpa_forward(q, k, v, bias=bias, scale=0.37, lib=lib),
           _torch_sdpa(q, k, v, attn_mask=bias, scale=0.37))


# ---- closed forms -------------------------------------------------------------------------

@pin
def closed_form_two_keys(lib):
    """With two keys the softmax is a logistic function: w0 = 1/(1+exp(x1-x0)), where
    x = scale·qᵀk + bias (arguments scale and bias)."""
    rng = _rng(21)
    q, k, v = _qkv(rng, 1, 1, 2, 1, 1, 4, 3)
    bias = np.array([[[[0.8, -1.3]]]])
    s = 0.5
    x0 = s * float(q[0, 0, 0] @ k[0, 0, 0]) + 0.8
    x1 = s * float(q[0, 0, 0] @ k[0, 1, 0]) - 1.3
    w0 = 1.0 / (1.0 + math.exp(x1 - x0))
    expect = w0 * v[0, 0, 0] + (1.0 - w0) * v[0, 1, 0]
    _close(oracle.sdpa_forward(q, k, v, bias=bias, scale=s, lib=lib)[0, 0, 0], expect)


@pin
def default_scale_uses_qk_dim(lib):
    """Argument scale: nothing means 1/√(qk_head_dim), even when v_head_dim differs."""
    q, k, v = _qkv(_rng(22), 1, 3, 4, 1, 1, 9, 4)
    _close(oracle.sdpa_forward(q, k, v, lib=lib), oracle.sdpa_forward(q, k, v, scale=1 / 3.0, lib=lib))


@pin
def rows_sum_to_one(lib):
    """The softmax weights of a row sum to one: with every value equal to 1 the output is 1,
    whatever the bias, mask, causal alignment and lengths."""
    rng = _rng(23)
    q, k, _ = _qkv(rng, 3, 5, 9, 4, 2, 8)
    v = np.ones((3, 9, 2, 5))
    mask = rng.random((3, 4, 5, 9)) < 0.7
    mask[..., 0] = True
    bias = 3.0 * rng.standard_normal((1, 4, 5, 9))
    out = oracle.sdpa_forward(q, k, v, bias=bias, mask=mask, is_causal=True, q_offset=[0, 2, 4],
                              kv_lengths=[9, 5, 7], lib=lib)
    _close(out, np.ones_like(out))


@pin
def weights_readout_is_a_distribution(lib):
    """With kv_len ≤ v_head_dim and value[j] = e_j, the output row is the weight row: it is
    non-negative, sums to one and is exactly zero on the keys that are not attended."""
    rng = _rng(24)
    Lk = 6
    q, k, _ = _qkv(rng, 1, 4, Lk, 1, 1, 8)
    v = np.eye(Lk)[None, :, None, :]
    mask = rng.random((1, 1, 4, Lk)) < 0.6
    mask[..., 1] = True
    w = oracle.sdpa_forward(q, k, v, mask=mask, lib=lib)[0, :, 0, :]
    assert (w >= 0).all()
    _close(w.sum(axis=-1), np.ones(4))
    assert (w[~mask[0, 0]] == 0).all()


@pin
def single_key_returns_its_value(lib):
    """With one attended key the weight is 1 and the output is that key's value: kv_lengths=1,
    and row 0 of is_causal=true (q_offset 0) sees only key 0."""
    q, k, v = _qkv(_rng(25), 2, 3, 5, 2, 1, 4, 6)
    out = oracle.sdpa_forward(q, k, v, kv_lengths=[1, 1], lib=lib)
    for b in range(2):
        for h in range(2):
            _close(out[b, :, h], np.broadcast_to(v[b, 0, 0], (3, 6)), 1e-15)
    out = oracle.sdpa_forward(q, k, v, is_causal=True, lib=lib)
    _close(out[:, 0, :, :], np.broadcast_to(v[:, 0:1, 0, :], (2, 2, 6)), 1e-15)


@pin
def identical_keys_average_values(lib):
    """All keys equal: every weight is 1/n over the n attended keys, so the output is the
    mean of their values (kv_lengths decides n)."""
    rng = _rng(26)
    q = rng.standard_normal((2, 3, 2, 4))
    k = np.broadcast_to(rng.standard_normal((1, 1, 1, 4)), (2, 6, 1, 4)).copy()
    v = rng.standard_normal((2, 6, 1, 5))
    out = oracle.sdpa_forward(q, k, v, kv_lengths=[4, 6], lib=lib)
    _close(out[0], np.broadcast_to(v[0, :4, 0].mean(0), (3, 2, 5)))
    _close(out[1], np.broadcast_to(v[1, :6, 0].mean(0), (3, 2, 5)))


# ---- equivalences the entry states ---------------------------------------------------------

@pin
def causal_equals_make_causal_mask(lib):
    """is_causal=true equals mask = make_causal_mask(query; dims=3) for equal lengths: the
    mask is true where key j ≤ query i."""
    q, k, v = _qkv(_rng(31), 2, 7, 7, 2, 2, 8)
    i = np.arange(7)[:, None]
    j = np.arange(7)[None, :]
    causal_mask = (j <= i)[None, None]
    _close(oracle.sdpa_forward(q, k, v, is_causal=True, lib=lib),
           oracle.sdpa_forward(q, k, v, mask=causal_mask, lib=lib))


@pin
def bottom_right_printed_example(lib):
    """Examples, KV-cache decoding: :bottom_right with kv_lengths [13,23,33,43] and 3 queries
    equals is_causal=true with q_offset [10,20,30,40] (sizes from the printed example)."""
    ex = json.load(open(os.path.join(GOLDEN, "printed_examples.json")))["examples"][3]
    D, H, Lq, B = ex["query"]
    _, Hk, Lk, _ = ex["key"]
    rng = _rng(32)
    q = rng.random((B, Lq, H, D))  # rand(Float32, ...) in the example: uniform [0, 1)
    k = rng.random((B, Lk, Hk, D))
    v = k  # k = v = rand(...) in the example
    a = oracle.sdpa_forward(q, k, v, is_causal="bottom_right", kv_lengths=ex["kv_lengths"], lib=lib)
    b = oracle.sdpa_forward(q, k, v, is_causal=True, q_offset=ex["equivalent_q_offset"],
                            kv_lengths=ex["kv_lengths"], lib=lib)
    _close(a, b, 0.0)
    assert a.shape == tuple(reversed(ex["output"]))
    # and the first new query attends exactly the keys 0 .. q_offset[b]
    c = oracle.sdpa_forward(q[:, :1], k, v, kv_lengths=np.array(ex["equivalent_q_offset"]) + 1, lib=lib)
    _close(a[:, :1], c)


@pin
def bottom_right_defaults_to_array_sizes(lib):
    """:bottom_right with no lengths: q_offset = kv_len - q_len of the arrays; with equal
    lengths it is the top-left mask."""
    q, k, v = _qkv(_rng(33), 2, 3, 8, 2, 2, 4)
    _close(oracle.sdpa_forward(q, k, v, is_causal="bottom_right", lib=lib),
           oracle.sdpa_forward(q, k, v, is_causal=True, q_offset=5, lib=lib), 0.0)
    q, k, v = _qkv(_rng(34), 2, 6, 6, 2, 2, 4)
    _close(oracle.sdpa_forward(q, k, v, is_causal="bottom_right", lib=lib),
           oracle.sdpa_forward(q, k, v, is_causal=True, lib=lib), 0.0)


@pin
def bottom_right_with_q_lengths(lib):
    """:bottom_right takes q_offset = kv_lengths - q_lengths per batch element when both are
    given; the last valid query then attends all kv_lengths keys."""
    q, k, v = _qkv(_rng(35), 2, 5, 9, 2, 2, 4)
    out = oracle.sdpa_forward(q, k, v, is_causal="bottom_right", q_lengths=[3, 5],
                              kv_lengths=[7, 9], lib=lib)
    ref = oracle.sdpa_forward(q, k, v, is_causal=True, q_offset=[4, 4], q_lengths=[3, 5],
                              kv_lengths=[7, 9], lib=lib)
    _close(out, ref, 0.0)
    full = oracle.sdpa_forward(q, k, v, kv_lengths=[7, 9], lib=lib)
    _close(out[0, 2], full[0, 2])
    _close(out[1, 4], full[1, 4])


@pin
def gqa_equals_repeated_heads(lib):
    """GQA paragraph: sharing key/value heads across query heads equals repeating each of them
    over its group of nheads/nkvheads consecutive query heads."""
    q, k, v = _qkv(_rng(36), 2, 4, 5, 6, 2, 4)
    _close(oracle.sdpa_forward(q, k, v, lib=lib),
           oracle.sdpa_forward(q, np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2), lib=lib))
    _close(oracle.sdpa_forward(q, k, v, kv_head_rule="interleaved", lib=lib),
           oracle.sdpa_forward(q, np.tile(k, (1, 1, 3, 1)), np.tile(v, (1, 1, 3, 1)), lib=lib))


@pin
def kv_lengths_equal_truncation(lib):
    """Argument kv_lengths: keys past kv_lengths[b] are not attended, which equals the call on
    arrays cut to that length (the padded-batch example)."""
    q, k, v = _qkv(_rng(37), 3, 4, 9, 2, 2, 4)
    lens = [3, 9, 6]
    out = oracle.sdpa_forward(q, k, v, kv_lengths=lens, lib=lib)
    for b, n in enumerate(lens):
        _close(out[b:b + 1], oracle.sdpa_forward(q[b:b + 1], k[b:b + 1, :n], v[b:b + 1, :n], lib=lib))
    # an integer applies to every batch element
    _close(oracle.sdpa_forward(q, k, v, kv_lengths=5, lib=lib),
           oracle.sdpa_forward(q, k[:, :5], v[:, :5], lib=lib))


@pin
def q_lengths_zero_rows(lib):
    """Argument q_lengths: the output is zero at the queries past q_lengths[b]; earlier rows
    are unchanged."""
    q, k, v = _qkv(_rng(38), 2, 6, 5, 2, 2, 4)
    out = oracle.sdpa_forward(q, k, v, q_lengths=[2, 6], lib=lib)
    full = oracle.sdpa_forward(q, k, v, lib=lib)
    assert (out[0, 2:] == 0).all()
    _close(out[0, :2], full[0, :2], 0.0)
    _close(out[1], full[1], 0.0)


@pin
def mask_causal_lengths_combine_by_and(lib):
    """mask, is_causal and kv_lengths combine: a key is attended only where all allow it, which
    equals one explicit mask that is their conjunction."""
    rng = _rng(39)
    q, k, v = _qkv(rng, 2, 6, 8, 2, 2, 4)
    mask = rng.random((2, 2, 6, 8)) < 0.7
    mask[..., 0] = True
    off = [1, 2]
    lens = [5, 8]
    i = np.arange(6)[:, None]
    j = np.arange(8)[None, :]
    combined = np.stack([mask[b] & (j <= off[b] + i)[None] & (j < lens[b])[None] for b in range(2)])
    _close(oracle.sdpa_forward(q, k, v, mask=mask, is_causal=True, q_offset=off, kv_lengths=lens, lib=lib),
           oracle.sdpa_forward(q, k, v, mask=combined, lib=lib))


@pin
def mask_equals_minus_infinity_bias(lib):
    """A false mask entry removes the key exactly as a bias of -infinity does; an all-true mask
    changes nothing."""
    rng = _rng(40)
    q, k, v = _qkv(rng, 2, 4, 7, 2, 2, 4)
    mask = rng.random((2, 2, 4, 7)) < 0.5
    mask[..., 3] = True
    bias = np.where(mask, 0.0, -np.inf)
    _close(oracle.sdpa_forward(q, k, v, mask=mask, lib=lib), oracle.sdpa_forward(q, k, v, bias=bias, lib=lib))
    _close(oracle.sdpa_forward(q, k, v, mask=np.ones((1, 1, 1, 1), bool), lib=lib),
           oracle.sdpa_forward(q, k, v, lib=lib), 0.0)


@pin
def bias_row_shift_invariance(lib):
    """Adding a constant per query row to the bias leaves the softmax unchanged."""
    rng = _rng(41)
    q, k, v = _qkv(rng, 2, 4, 6, 2, 2, 4)
    bias = rng.standard_normal((2, 2, 4, 6))
    shift = rng.standard_normal((2, 2, 4, 1)) * 5
    _close(oracle.sdpa_forward(q, k, v, bias=bias, lib=lib),
           oracle.sdpa_forward(q, k, v, bias=bias + shift, lib=lib), 1e-11)


@pin
def bias_is_per_head_and_batch(lib):
    """The bias is indexed by head and batch: a bias that differs only in head 1 / batch 1
    changes only those output rows, and a bias of a single key row equals a large logit."""
    rng = _rng(42)
    q, k, v = _qkv(rng, 2, 3, 5, 2, 2, 4)
    bias = np.zeros((2, 2, 3, 5))
    bias[1, 1, :, 2] = 80.0  # weight of key 2 becomes ~1 for batch 1, head 1
    out = oracle.sdpa_forward(q, k, v, bias=bias, lib=lib)
    ref = oracle.sdpa_forward(q, k, v, lib=lib)
    _close(out[0], ref[0], 0.0)
    _close(out[1, :, 0], ref[1, :, 0], 0.0)
    _close(out[1, :, 1], np.broadcast_to(v[1, 2, 1], (3, 4)), 1e-9)


@pin
def scale_equivalence(lib):
    """Argument scale multiplies qᵀk: scaling the query by a equals scaling `scale` by a."""
    q, k, v = _qkv(_rng(43), 2, 4, 6, 2, 2, 4)
    _close(oracle.sdpa_forward(2.5 * q, k, v, scale=0.3, lib=lib),
           oracle.sdpa_forward(q, k, v, scale=0.75, lib=lib))


@pin
def empty_row_is_nan_and_padding_wins(lib):
    """A query that attends to no key has a NaN output (fused-implementation paragraph); a
    query past q_lengths is zero even then."""
    q, k, v = _qkv(_rng(44), 1, 3, 4, 1, 1, 4)
    mask = np.ones((1, 1, 3, 4), bool)
    mask[0, 0, 1, :] = False
    mask[0, 0, 2, :] = False
    out = oracle.sdpa_forward(q, k, v, mask=mask, q_lengths=[2], lib=lib)
    assert np.isfinite(out[0, 0]).all()
    assert np.isnan(out[0, 1]).all()
    assert (out[0, 2] == 0).all()
    # a negative causal offset leaves the first rows without keys
    out = oracle.sdpa_forward(q, k, v, is_causal=True, q_offset=-2, lib=lib)
    assert np.isnan(out[0, :2]).all() and np.isfinite(out[0, 2]).all()


@pin
def printed_example_shapes(lib):
    """Examples: the output has size (v_head_dim, nheads, q_len, batch) for the plain, GQA
    and padded calls."""
    ex = json.load(open(os.path.join(GOLDEN, "printed_examples.json")))["examples"]
    rng = _rng(45)
    for e in ex[:3]:
        qs, ks, vs = (tuple(reversed(e[n])) for n in ("query", "key", "value"))
        out = oracle.sdpa_forward(rng.random(qs), rng.random(ks), rng.random(vs),
                                  kv_lengths=e.get("kv_lengths"), lib=lib)
        assert out.shape == tuple(reversed(e["output"]))
        assert np.isfinite(out).all()


# ---- rotary position embedding (the Keras thread's "rotary embeddings") ----------------------

@pin
def rope_two_dims_is_a_plane_rotation(lib):
    """With d = 2 the single pair rotates by the position itself (frequency base^0 = 1):
    the textbook plane rotation."""
    x = _rng(91).standard_normal((5, 3, 2))
    pos = np.array([0, 1, 7, -3, 1000])
    out = oracle.rope(x, pos, lib=lib)
    c, s_ = np.cos(pos)[:, None], np.sin(pos)[:, None]
    _close(out[..., 0], x[..., 0] * c - x[..., 1] * s_)
    _close(out[..., 1], x[..., 1] * c + x[..., 0] * s_)


@pin
def rope_is_a_rotation_by_relative_position(lib):
    """Each pair is rotated, so norms are kept, position 0 is the identity, rotating by -p undoes
    p, and q.k after the embedding depends only on the difference of the two positions (the
    reason the embedding is applied to both query and key)."""
    rng = _rng(92)
    x = rng.standard_normal((6, 4, 64))
    pos = rng.integers(-5000, 5000, size=6)
    out = oracle.rope(x, pos, lib=lib)
    _close(np.linalg.norm(out, axis=-1), np.linalg.norm(x, axis=-1))
    _close(oracle.rope(x, np.zeros(6), lib=lib), x, 0.0)
    _close(oracle.rope(out, -pos, lib=lib), x, 1e-11)
    q, k = rng.standard_normal((2, 1, 2, 128))
    for m, n, shift in ((3, 11, 100), (4000, 17, -2000), (0, 0, 12345)):
        a = oracle.rope(q, [m], lib=lib)[0] @ oracle.rope(k, [n], lib=lib)[0].T
        b = oracle.rope(q, [m + shift], lib=lib)[0] @ oracle.rope(k, [n + shift], lib=lib)[0].T
        _close(a, b, 1e-9)


@pin
def rope_pairs_halves_with_geometric_frequencies(lib):
    """A unit vector along dimension c < d/2 moves only within the plane of c and c + d/2, and
    the angle measured at position 1 falls geometrically with c, from 1 radian, by the factor
    base^(-2/d)."""
    d, base = 16, 500.0
    angles = []
    for c in range(d // 2):
        e = np.zeros((1, 1, d))
        e[0, 0, c] = 1.0
        out = oracle.rope(e, [1], base=base, lib=lib)[0, 0]
        others = np.delete(out, [c, c + d // 2])
        _close(others, np.zeros(d - 2), 0.0)
        angles.append(math.atan2(out[c + d // 2], out[c]))
    angles = np.array(angles)
    _close(angles[0], 1.0, 1e-14)
    _close(angles[1:] / angles[:-1], np.full(d // 2 - 1, base ** (-2 / d)), 1e-12)


# ---- the row log-sum-exp (the softmax's normaliser) ----------------------------------------

@pin
def lse_is_torch_logsumexp_of_the_masked_logits(lib):
    """oracle.sdpa_forward_lse's lse is PyTorch's float64 logsumexp over each row's attended
    logits (scale q.k + bias, causal with offsets, lengths, GQA through repeated heads), +inf for
    a row with no key and for padding rows; the output equals the plain forward's; and the
    weights exp(logit - lse) of a row add up to 1."""
    rng = _rng(91)
    B, Lq, Lk, H, Hkv, D = 2, 9, 12, 4, 2, 8
    q, k, v = _qkv(rng, B, Lq, Lk, H, Hkv, D)
    bias = rng.standard_normal((1, H, Lq, Lk))
    kw = dict(bias=bias, is_causal=True, q_offset=[2, -3], q_lengths=[9, 6], kv_lengths=[12, 10], scale=0.4)
    out, lse = oracle.sdpa_forward_lse(q, k, v, lib=lib, **kw)
    _close(out, oracle.sdpa_forward(q, k, v, lib=lib, **kw), 0.0)
    kr = np.repeat(k, H // Hkv, axis=2)
    logits = 0.4 * np.einsum("bihd,bjhd->bhij", q, kr) + bias
    i = np.arange(Lq)[:, None]
    j = np.arange(Lk)[None, :]
    for b, (off, ql, kl) in enumerate(zip([2, -3], [9, 6], [12, 10])):
        allowed = (j <= off + i) & (j < kl) & (i < ql)
        x = torch.from_numpy(np.where(allowed[None], logits[b], -np.inf))
        want = torch.logsumexp(x, dim=-1).numpy()
        want = np.where(np.isneginf(want), np.inf, want)  # no key: +inf
        want[:, ql:] = np.inf  # padding rows: +inf
        assert np.array_equal(np.isinf(lse[b]), np.isinf(want))
        fin = np.isfinite(want)
        _close(lse[b][fin], want[fin], 1e-12)
        w = np.where(allowed[None], np.exp(logits[b] - lse[b][..., None]), 0.0)
        rows = fin
        _close(w.sum(-1)[rows], np.ones(int(rows.sum())), 1e-12)


# ---- with weights and fdrop (the entry's "See also"; argument fdrop) -------------------------

@pin
def with_weights_equals_torch_softmax(lib):
    """The materialized weights are PyTorch's float64 softmax of scale*q.k + bias over the
    attended keys (masked logits at -inf; GQA by repeated heads), in the page's (kv_len,
    q_len, nheads, batch) order, and the output is those weights times V."""
    rng = _rng(81)
    q, k, v = _qkv(rng, 2, 5, 7, 4, 2, 6, 3)
    bias = rng.standard_normal((4, 5, 7))
    mask = rng.random((2, 4, 5, 7)) < 0.7
    mask[..., 0] = True
    out, w = oracle.sdpa_forward_with_weights(q, k, v, bias=bias, mask=mask, scale=0.6, lib=lib)
    kk = np.repeat(k, 2, axis=2)
    logits = 0.6 * np.einsum("bihc,bjhc->bhij", q, kk) + bias[None]
    logits = torch.from_numpy(np.where(mask, logits, -np.inf))
    want = torch.softmax(logits, dim=-1).numpy()
    _close(w, want)
    _close(out, np.einsum("bhij,bjhe->bihe", w, np.repeat(v, 2, axis=2)))


@pin
def with_weights_empty_and_padding_rows(lib):
    """A row with no attended key has NaN weights and output; a row past q_lengths has zero
    weights and output; causal rows put no weight past q_offset + i."""
    rng = _rng(82)
    q, k, v = _qkv(rng, 2, 4, 6, 2, 2, 4)
    out, w = oracle.sdpa_forward_with_weights(q, k, v, is_causal=True, q_offset=[1, -2],
                                              q_lengths=[3, 4], lib=lib)
    assert np.isnan(w[1, :, :2]).all() and np.isnan(out[1, :2]).all()
    assert (w[0, :, 3] == 0).all() and (out[0, 3] == 0).all()
    i = np.arange(4)[:, None]
    j = np.arange(6)[None, :]
    # softmax weights are positive exactly on the attended keys j <= q_offset + i
    assert ((w[0, :, :3] > 0) == (j <= 1 + i)[None, :3]).all()
    assert ((w[1, :, 2:] > 0) == (j <= -2 + i)[None, 2:]).all()
    _close(np.nansum(w[0, :, :3], axis=-1), np.ones((2, 3)))


@pin
def dropout_keeps_one_minus_p_unbiased(lib):
    """fdrop as dropout: each weight is kept with probability 1 - p and then divided by 1 - p,
    so the kept fraction is 1 - p (checked within 5 standard deviations on 40,000 weights) and
    the average over seeds is the undropped weight. The output is the dropped weights times
    V. p = 0 changes nothing; another seed gives another pattern."""
    rng = _rng(83)
    q, k, v = _qkv(rng, 2, 40, 50, 10, 5, 8)
    o0, w0 = oracle.sdpa_forward_with_weights(q, k, v, lib=lib)
    o1, w1 = oracle.sdpa_forward_with_weights(q, k, v, drop_p=0.0, seed=99, lib=lib)
    _close(w0, w1, 0.0)
    _close(o0, o1, 0.0)
    p = 0.3
    out, w = oracle.sdpa_forward_with_weights(q, k, v, drop_p=p, seed=7, lib=lib)
    kept = w != 0
    n = kept.size
    assert abs(kept.mean() - (1 - p)) < 5 * math.sqrt(p * (1 - p) / n)
    _close(w[kept], w0[kept] / (1 - p), 1e-15)
    _close(out, np.einsum("bhij,bjhe->bihe", w, np.repeat(v, 2, axis=2)))
    # neighbouring weights draw independently, also the four that share one 64-bit hash
    a, c = kept[..., :-1].ravel(), kept[..., 1:].ravel()
    both = (a & c).mean()
    assert abs(both - (1 - p) ** 2) < 5 * math.sqrt((1 - p) ** 2 * (1 - (1 - p) ** 2) / a.size)
    _, w2 = oracle.sdpa_forward_with_weights(q, k, v, drop_p=p, seed=8, lib=lib)
    assert ((w2 != 0) != kept).mean() > 0.3
    acc = np.zeros((1, 10, 4, 50))
    for s in range(300):
        acc += oracle.sdpa_forward_with_weights(q[:1, :4], k[:1], v[:1], drop_p=p, seed=1000 + s, lib=lib)[1]
    ref = w0[:1, :, :4]
    sd = np.sqrt(ref ** 2 * p / (1 - p) / 300)
    assert (np.abs(acc / 300 - ref) <= 5 * sd + 1e-12).all()
    try:
        oracle.sdpa_forward_with_weights(q, k, v, drop_p=1.0, lib=lib)
    except oracle.OracleError:
        pass
    else:
        raise AssertionError("drop probability 1 accepted")


# ---- the fused gradient (paragraph "Fused implementation") -----------------------------------

def _loss(q, k, v, dout, lib, **kw):
    """sum(dout * out) over the rows that attend some key (NaN rows take no part)."""
    out = oracle.sdpa_forward(q, k, v, lib=lib, **kw)
    return float(np.nansum(dout * out))


def _central(f, x, h=1e-6):
    """Central differences of the scalar f with respect to every element of x (in place)."""
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        old = x[idx]
        x[idx] = old + h
        up = f()
        x[idx] = old - h
        down = f()
        x[idx] = old
        g[idx] = (up - down) / (2 * h)
    return g


@pin
def backward_finite_differences(lib):
    """dq, dk, dv and dscale are the derivatives of sum(dout * out): checked element by element
    against central differences of the (separately pinned) forward, with GQA, dv != dqk,
    causal offsets, kv_lengths, q_lengths, a mask and a row that attends no key."""
    rng = _rng(71)
    q, k, v = _qkv(rng, 2, 4, 5, 4, 2, 3, 2)
    dout = rng.standard_normal((2, 4, 4, 2))
    mask = rng.random((1, 4, 4, 5)) < 0.7
    cases = (dict(is_causal=True, q_offset=[1, -1], kv_lengths=[5, 3], scale=0.7),
             dict(mask=mask, q_lengths=[3, 4], kv_lengths=[4, 5]),
             dict(is_causal="bottom_right", q_lengths=[2, 4], kv_lengths=[4, 2]))
    for kw in cases:
        dq, dk, dv, ds = oracle.sdpa_backward(q, k, v, dout, lib=lib, **kw)
        f = lambda: _loss(q, k, v, dout, lib, **kw)
        _close(dq, _central(f, q), 1e-6)
        _close(dk, _central(f, k), 1e-6)
        _close(dv, _central(f, v), 1e-6)
        s0 = kw.get("scale", 1 / math.sqrt(3))
        g = lambda s: _loss(q, k, v, dout, lib, **{**kw, "scale": s})
        _close(ds, (g(s0 + 1e-6) - g(s0 - 1e-6)) / 2e-6, 1e-6)


@pin
def backward_equals_torch_autograd(lib):
    """PyTorch's float64 autograd of its scaled_dot_product_attention (GQA by repeating each
    key/value head over its group of query heads, which autograd sums back; causal; a
    boolean mask)."""
    rng = _rng(72)
    q, k, v = _qkv(rng, 2, 9, 9, 6, 2, 8, 5)
    dout = rng.standard_normal((2, 9, 6, 5))
    mask = rng.random((2, 6, 9, 9)) < 0.8
    mask[..., 0] = True  # every row keeps a key
    for kw, tkw in ((dict(is_causal=True), dict(is_causal=True)),
                    (dict(mask=mask), dict(attn_mask=torch.from_numpy(mask)))):
        tq, tk, tv = (torch.from_numpy(a.copy()).requires_grad_(True) for a in (q, k, v))
        kk = tk.repeat_interleave(3, dim=2).permute(0, 2, 1, 3)
        vv = tv.repeat_interleave(3, dim=2).permute(0, 2, 1, 3)
        out = torch.nn.functional.scaled_dot_product_attention(tq.permute(0, 2, 1, 3), kk, vv, **tkw)
        out.permute(0, 2, 1, 3).backward(torch.from_numpy(dout))
        dq, dk, dv, _ = oracle.sdpa_backward(q, k, v, dout, lib=lib, **kw)
        _close(dq, tq.grad.numpy())
        _close(dk, tk.grad.numpy())
        _close(dv, tv.grad.numpy())


@pin
def backward_invariants(lib):
    """The weights of a row sum to one, so its logit gradients sum to zero: the key gradients
    of a (batch, kv head) sum to zero, the value gradients sum to the dout of the rows that
    attend some key, and scale * dscale = sum of q . dq."""
    rng = _rng(73)
    q, k, v = _qkv(rng, 2, 6, 7, 4, 2, 5, 3)
    dout = rng.standard_normal((2, 6, 4, 3))
    kw = dict(is_causal=True, q_offset=[0, -2], scale=0.45)
    dq, dk, dv, ds = oracle.sdpa_backward(q, k, v, dout, lib=lib, **kw)
    _close(dk.sum(axis=1), np.zeros((2, 2, 5)))
    rows = np.ones((2, 6), dtype=bool)
    rows[1, :2] = False  # offset -2: the first two rows of batch 1 attend no key
    want = np.stack([np.stack([dout[b][rows[b]][:, 2 * g:2 * g + 2].sum(axis=(0, 1)) for g in range(2)])
                     for b in range(2)])
    _close(dv.sum(axis=1), want)
    _close(0.45 * ds, float((q * dq).sum()))


@pin
def backward_excludes_empty_and_padding_rows(lib):
    """A row with no attended key (NaN output) and a row past q_lengths (zero output) take no
    part: their dq is zero and their dout changes nothing."""
    rng = _rng(74)
    q, k, v = _qkv(rng, 2, 5, 6, 2, 2, 4)
    dout = rng.standard_normal((2, 5, 2, 4))
    kw = dict(q_lengths=[3, 5], kv_lengths=[6, 0])
    a = oracle.sdpa_backward(q, k, v, dout, lib=lib, **kw)
    _close(a[0][0, 3:], np.zeros((2, 2, 4)), 0.0)
    _close(a[0][1], np.zeros((5, 2, 4)), 0.0)
    d2 = dout.copy()
    d2[0, 3:] = 100.0
    d2[1] = -7.0
    b = oracle.sdpa_backward(q, k, v, d2, lib=lib, **kw)
    for x, y in zip(a[:3], b[:3]):
        _close(x, y, 0.0)
    assert a[3] == b[3]


# ---- packed sequences (keywords q_segments, kv_segments, maxlen; paragraph "Packed sequences")

def _brute_packed(q, k, v, qs, ks, causal=False, q_offset=None, q_lengths=None, kv_lengths=None):
    """Pure-Python packed attention on tiny inputs: every (segment, query row, head) with
    math.exp over its own segment's keys; kv head h // (H/Hkv)."""
    Lq, H, D = q.shape
    Hkv, Dv = k.shape[1], v.shape[2]
    out = np.zeros((Lq, H, Dv))
    q0 = k0 = 0
    for s in range(len(qs)):
        ql = qs[s] if q_lengths is None else q_lengths[s]
        kl = ks[s] if kv_lengths is None else kv_lengths[s]
        off = 0 if q_offset is None else q_offset[s]
        if causal == "bottom_right":
            off = kl - ql
        for i in range(qs[s]):
            for h in range(H):
                if i >= ql:
                    continue
                g = h // (H // Hkv)
                keys = [j for j in range(ks[s]) if j < kl and (not causal or j <= off + i)]
                if not keys:
                    out[q0 + i, h] = float("nan")
                    continue
                x = [sum(q[q0 + i, h, c] * k[k0 + j, g, c] for c in range(D)) / math.sqrt(D) for j in keys]
                m = max(x)
                w = [math.exp(t - m) for t in x]
                z = sum(w)
                for e in range(Dv):
                    out[q0 + i, h, e] = sum(w[n] * v[k0 + j, g, e] for n, j in enumerate(keys)) / z
        q0 += qs[s]
        k0 += ks[s]
    return out


@pin
def packed_brute_force(lib):
    """Each query segment attends its own key/value segment only, as a batch element of a
    padded batch would, with is_causal, q_offset, q_lengths and kv_lengths taken per segment;
    checked against pure-Python loops (GQA, unequal q/kv segments, an empty segment, a
    query row with no key, head dims 3 and 2)."""
    rng = _rng(61)
    qs, ks = [3, 0, 4, 2], [2, 3, 5, 1]
    q = rng.standard_normal((sum(qs), 4, 3))
    k = rng.standard_normal((sum(ks), 2, 3))
    v = rng.standard_normal((sum(ks), 2, 2))
    for kw in (dict(), dict(causal=True, q_offset=[0, 1, 1, -1]),
               dict(causal=True, q_offset=[1, 0, 2, 0], q_lengths=[2, 0, 4, 1], kv_lengths=[2, 1, 4, 1]),
               dict(causal="bottom_right", q_lengths=[3, 0, 3, 2], kv_lengths=[2, 3, 4, 1])):
        want = _brute_packed(q, k, v, qs, ks, **kw)
        got = oracle.sdpa_forward_packed(q, k, v, qs, ks, is_causal=kw.get("causal", False),
                                         q_offset=kw.get("q_offset", 0), q_lengths=kw.get("q_lengths"),
                                         kv_lengths=kw.get("kv_lengths"), lib=lib)
        assert (np.isnan(got) == np.isnan(want)).all()
        _close(np.nan_to_num(got), np.nan_to_num(want))


@pin
def packed_first_query_of_each_causal_segment(lib):
    """With is_causal and q_offset 0, the first query of a segment sees only the segment's
    first key, so its output is that key's value (kv_segments defaulting to q_segments)."""
    rng = _rng(62)
    segs = [5, 12, 3, 1, 7]
    x = rng.standard_normal((sum(segs), 2, 6))
    y = oracle.sdpa_forward_packed(x, x, x, segs, is_causal=True, lib=lib)
    start = np.cumsum([0] + segs[:-1])
    _close(y[start], x[start], 1e-15)


@pin
def packed_segments_are_isolated(lib):
    """Changing the keys and values of one segment changes that segment's output only."""
    rng = _rng(63)
    qs, ks = [6, 9, 4], [7, 5, 8]
    q = rng.standard_normal((sum(qs), 4, 8))
    k = rng.standard_normal((sum(ks), 2, 8))
    v = rng.standard_normal((sum(ks), 2, 8))
    a = oracle.sdpa_forward_packed(q, k, v, qs, ks, lib=lib)
    k2, v2 = k.copy(), v.copy()
    k2[7:12] = rng.standard_normal((5, 2, 8))
    v2[7:12] = rng.standard_normal((5, 2, 8))
    b = oracle.sdpa_forward_packed(q, k2, v2, qs, ks, lib=lib)
    _close(a[:6], b[:6], 0.0)
    _close(a[15:], b[15:], 0.0)
    assert np.abs(a[6:15] - b[6:15]).min() > 0


@pin
def packed_equals_torch_per_segment(lib):
    """Segment by segment, packed attention is PyTorch's float64 routine on that segment
    alone (GQA by repeated heads, causal with per-segment q_offset as a boolean mask)."""
    rng = _rng(64)
    qs, ks, off = [33, 17, 64], [40, 17, 70], [7, 0, 6]
    q = rng.standard_normal((sum(qs), 6, 16))
    k = rng.standard_normal((sum(ks), 2, 16))
    v = rng.standard_normal((sum(ks), 2, 12))
    got = oracle.sdpa_forward_packed(q, k, v, qs, ks, is_causal=True, q_offset=off, lib=lib)
    q0 = k0 = 0
    for s in range(3):
        qq = q[None, q0:q0 + qs[s]]
        kk = np.repeat(k[None, k0:k0 + ks[s]], 3, axis=2)
        vv = np.repeat(v[None, k0:k0 + ks[s]], 3, axis=2)
        i = np.arange(qs[s])[:, None]
        j = np.arange(ks[s])[None, :]
        want = _torch_sdpa(qq, kk, vv, attn_mask=(j <= off[s] + i))
        _close(got[q0:q0 + qs[s]], want[0])
        q0 += qs[s]
        k0 += ks[s]


@pin
def packed_printed_example_and_errors(lib):
    """Examples: x of size (16, 8, 20) with q_segments [5, 12, 3] and is_causal keeps its size.
    The segment lengths must add up to the array lengths, and maxlen must be at least every
    segment."""
    ex = json.load(open(os.path.join(GOLDEN, "printed_examples.json")))["examples"][4]
    x = _rng(65).random(tuple(reversed(ex["query"])))
    y = oracle.sdpa_forward_packed(x, x, x, ex["q_segments"], is_causal=ex["is_causal"], maxlen=12, lib=lib)
    assert y.shape == tuple(reversed(ex["output"])) and np.isfinite(y).all()
    for bad in (dict(q_segments=[5, 12, 2]), dict(q_segments=[5, 12, 3], maxlen=11),
                dict(q_segments=[5, 12, 3], kv_segments=[5, 13, 3]), dict(q_segments=[6, -1, 15])):
        try:
            oracle.sdpa_forward_packed(x, x, x, lib=lib, **bad)
        except oracle.OracleError:
            continue
        raise AssertionError(f"accepted {bad}")


# ---- cache update and decode ----------------------------------------------------------------

@pin
def cache_update_writes_only_the_new_rows(lib):
    """Keras issue on MultiHeadAttention, cache_update_index: the new keys/values are written
    at the given position of each sequence; every other cache entry is unchanged."""
    rng = _rng(51)
    cache = rng.standard_normal((3, 10, 2, 4))
    new = rng.standard_normal((3, 2, 2, 4))
    idx = [0, 5, 8]
    out = oracle.cache_update_at_index(cache, new, idx, lib=lib)
    expect = cache.copy()
    for b, i in enumerate(idx):
        expect[b, i:i + 2] = new[b]
    _close(out, expect, 0.0)
    try:
        oracle.cache_update_at_index(cache, new, [0, 5, 9], lib=lib)
    except oracle.OracleError:
        pass
    else:
        raise AssertionError("an index past capacity - n_new must be rejected")


@pin
def decode_equals_attention_over_the_grown_cache(lib):
    """Decoding example: after writing the new key/value at index[b], :bottom_right attention
    of one new query equals plain attention over the index[b] + 1 keys of the cache."""
    rng = _rng(52)
    B, cap, H, Hkv, D = 3, 12, 4, 2, 8
    q = rng.standard_normal((B, 1, H, D))
    kn, vn = rng.standard_normal((B, 1, Hkv, D)), rng.standard_normal((B, 1, Hkv, D))
    kc, vc = rng.standard_normal((B, cap, Hkv, D)), rng.standard_normal((B, cap, Hkv, D))
    idx = np.array([0, 6, 11])
    out, kc2, vc2 = oracle.sdpa_decode_with_cache(q, kn, vn, kc, vc, idx, lib=lib)
    for b in range(B):
        n = idx[b] + 1
        kk = np.concatenate([kc[b:b + 1, :idx[b]], kn[b:b + 1]], axis=1)
        vv = np.concatenate([vc[b:b + 1, :idx[b]], vn[b:b + 1]], axis=1)
        _close(out[b:b + 1], oracle.sdpa_forward(q[b:b + 1], kk, vv, lib=lib))
        _close(kc2[b, :n], kk[0], 0.0)
    # several new queries: the t-th attends the keys up to index[b] + t
    q3 = rng.standard_normal((B, 3, H, D))
    kn3, vn3 = rng.standard_normal((B, 3, Hkv, D)), rng.standard_normal((B, 3, Hkv, D))
    idx3 = np.array([0, 4, 9])
    out3, kc3, vc3 = oracle.sdpa_decode_with_cache(q3, kn3, vn3, kc, vc, idx3, lib=lib)
    for b in range(B):
        for t in range(3):
            n = idx3[b] + t + 1
            _close(out3[b:b + 1, t:t + 1],
                   oracle.sdpa_forward(q3[b:b + 1, t:t + 1], kc3[b:b + 1, :n], vc3[b:b + 1, :n], lib=lib))


# ---- block classification --------------------------------------------------------------------

def _decode_info(info, H, Lq, Lk, bq, bk):
    """Rebuild the dense mask from the classes and the packed partial bits."""
    m = np.zeros((H, Lq, Lk), dtype=np.uint8)
    nqb, nkb = info["cls"].shape[1:]
    for h in range(H):
        for qb in range(nqb):
            for kb in range(nkb):
                c = info["cls"][h, qb, kb]
                r0, c0 = qb * bq, kb * bk
                r1, c1 = min(Lq, r0 + bq), min(Lk, c0 + bk)
                if c == 2:
                    m[h, r0:r1, c0:c1] = 1
                elif c == 1:
                    words = info["bits"][h, qb, kb]
                    for r in range(r1 - r0):
                        for cc in range(c1 - c0):
                            m[h, r0 + r, c0 + cc] = (words[r, cc // 32] >> (cc % 32)) & 1
    return m


@pin
def block_info_hand_built_classes(lib):
    """Splash-attention mask info (JAX pull request "Support dynamic masks in splash
    attention"): a block with no attended cell is empty, one with all cells attended is
    full, any other is partial; the per-row list holds the non-empty blocks in order."""
    H, Lq, Lk, b = 1, 8, 12, 4
    m = np.zeros((H, Lq, Lk), np.uint8)
    m[0, 0:4, 4:8] = 1          # (0,1) full
    m[0, 1, 9] = 1              # (0,2) partial
    m[0, 4:8, 0:4] = 1
    m[0, 6, 2] = 0              # (1,0) partial
    m[0, 4:8, 8:12] = 1         # (1,2) full
    info = oracle.block_mask_info(m, b, b, lib=lib)
    assert info["cls"].tolist() == [[[0, 2, 1], [1, 0, 2]]]
    assert info["count"].tolist() == [[2, 2]]
    assert [int(x) for x in info["list"][0, 0, :2]] == [1 | (2 << 30), 2 | (1 << 30)]
    assert [int(x) for x in info["list"][0, 1, :2]] == [0 | (1 << 30), 2 | (2 << 30)]
    assert int(info["bits"][0, 0, 2, 1, 0]) == 1 << 1
    assert int(info["bits"][0, 1, 0, 2, 0]) == 0b1011


@pin
def block_info_round_trip_ragged(lib):
    """Brute force: on random masks with ragged edges, the classes count the attended cells
    correctly and the packed partial bits rebuild the mask exactly."""
    rng = _rng(53)
    H, Lq, Lk, bq, bk = 2, 37, 70, 16, 32
    m = (rng.random((H, Lq, Lk)) < 0.5).astype(np.uint8)
    m[:, :16, :32] = 0
    m[:, 16:32, 32:64] = 1
    m[:, 32:37, 64:70] = 1  # a full block at the ragged corner
    info = oracle.block_mask_info(m, bq, bk, lib=lib)
    np.testing.assert_array_equal(_decode_info(info, H, Lq, Lk, bq, bk), m)
    for h in range(H):
        for qb in range(info["cls"].shape[1]):
            for kb in range(info["cls"].shape[2]):
                blk = m[h, qb * bq:(qb + 1) * bq, kb * bk:(kb + 1) * bk]
                want = 0 if blk.sum() == 0 else (2 if blk.all() else 1)
                assert info["cls"][h, qb, kb] == want
            n = info["count"][h, qb]
            assert n == int((info["cls"][h, qb] != 0).sum())
            kbs = [int(x) & ((1 << 30) - 1) for x in info["list"][h, qb, :n]]
            assert kbs == sorted(kbs) and all(info["cls"][h, qb, kb] != 0 for kb in kbs)
