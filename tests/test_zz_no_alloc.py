"""The decode entry point for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc (a plug-in inside a framework that owns all
device memory, or a decode loop that must not touch the allocator mid-run), so they cannot pass
the workspace sdpa_decode_with_cache needs. sdpa_decode_with_cache_static takes the same
arguments minus the workspace and keeps its scratch in a fixed array inside the library;
sdpa_read_static_status reads (and clears) the device status word that sits in that array.

These tests call both through the C ABI. They check the static entry against the oracle and
against sdpa_decode_with_cache on the same inputs, on two calls in a row (the array keeps the
previous call's contents), at a small size and at the full KV-cache decode workload; that an
out-of-range cache index gives NaN rows and a status the caller can read; and that a call too
large for the array is refused before anything runs. The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sdpa_inputs as si
from parity import assert_matches, f64

pytestmark = pytest.mark.gpu

sdpa = pytest.importorskip("head_scaled_dot_sdpa_b200")
DEV = "cuda"
TOL = 1e-2  # bf16 outputs, as in the other decode parity tests

fn = sdpa.lib.sdpa_decode_with_cache_static
fn.argtypes = [ctypes.POINTER(sdpa.Params)] + [ctypes.c_void_p] * 8
fn.restype = ctypes.c_int
read_status = sdpa.lib.sdpa_read_static_status
read_status.argtypes = [ctypes.c_void_p]
read_status.restype = ctypes.c_int


def _small():
    w = si.scaled(si.KV_CACHE_DECODE, batch=6, capacity=1500, kv_len=1500, kv_len_min=1, kv_len_max=1500)
    return si.decode_inputs(w)


def _params(q, k_cache, v_cache):
    p = sdpa.Params()
    p.dtype = sdpa.SDPA_BF16
    p.batch, p.q_len, p.kv_len = q.shape[0], q.shape[1], k_cache.shape[1]
    p.nheads, p.nkvheads, p.dqk, p.dv = q.shape[2], k_cache.shape[2], q.shape[3], v_cache.shape[3]
    p.scale = float("nan")
    p.causal = sdpa.SDPA_CAUSAL_BOTTOM_RIGHT
    return p


def _call_static(q, kn, vn, kc, vc, idx, out):
    p = _params(q, kc, vc)
    stream = torch.cuda.current_stream().cuda_stream
    rc = fn(ctypes.byref(p), q.data_ptr(), kn.data_ptr(), vn.data_ptr(), kc.data_ptr(), vc.data_ptr(),
            idx.data_ptr(), out.data_ptr(), stream)
    torch.cuda.synchronize()
    return rc


def _status():
    return read_status(torch.cuda.current_stream().cuda_stream)


def _check_against_workspace_and_oracle(d, rows):
    q, kn, vn = d["q"].to(DEV), d["k_new"].to(DEV), d["v_new"].to(DEV)
    idx = d["index"].to(DEV)
    kc_ref, vc_ref = d["k_cache"].to(DEV), d["v_cache"].to(DEV)
    ref = sdpa.sdpa_decode_with_cache(q, kn, vn, kc_ref, vc_ref, idx)
    torch.cuda.synchronize()
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    kc, vc = d["k_cache"].to(DEV), d["v_cache"].to(DEV)
    index = d["index"].numpy()
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        rc = _call_static(q, kn, vn, kc, vc, idx, out)
        assert rc == sdpa.SDPA_OK, sdpa.lib.sdpa_last_error().decode()
        assert _status() == sdpa.SDPA_OK
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= TOL, f"call {call}: max-abs difference to sdpa_decode_with_cache {err}"
        assert torch.equal(kc, kc_ref) and torch.equal(vc, vc_ref)
        got = out.cpu()
        for b in rows:
            want, _, _ = oracle.sdpa_decode_with_cache(
                f64(d["q"][b:b + 1]), f64(d["k_new"][b:b + 1]), f64(d["v_new"][b:b + 1]),
                f64(d["k_cache"][b:b + 1]), f64(d["v_cache"][b:b + 1]), index[b:b + 1])
            assert_matches(got[b:b + 1], want, TOL, f"static call {call}, sequence {b}")


def test_static_scratch_matches_oracle_and_workspace_entry_point():
    d = _small()
    _check_against_workspace_and_oracle(d, range(d["q"].shape[0]))


def test_static_scratch_full_kv_cache_decode_workload():
    # the full KV-cache decode workload (64 sequences, capacity 8192) fits the 40 MiB array
    w = si.KV_CACHE_DECODE
    d = si.decode_inputs(w)
    p = _params(d["q"], d["k_cache"], d["v_cache"])
    assert sdpa.lib.sdpa_workspace_size(ctypes.byref(p)) <= 40 << 20
    _check_against_workspace_and_oracle(d, [0, 21, 42, 63])


def test_static_scratch_bad_index_gives_nan_rows_and_a_readable_status():
    d = _small()
    q, kn, vn = d["q"].to(DEV), d["k_new"].to(DEV), d["v_new"].to(DEV)
    kc, vc = d["k_cache"].to(DEV), d["v_cache"].to(DEV)
    index = d["index"].numpy().copy()
    cap = d["k_cache"].shape[1]
    index[2] = cap  # one past the last row that a 1-token write may start at
    out = torch.zeros_like(q)
    rc = _call_static(q, kn, vn, kc, vc, torch.from_numpy(index).to(DEV), out)
    assert rc == sdpa.SDPA_OK  # the index is on the device: found there, not on the host
    assert _status() == sdpa.SDPA_ERR_DEVICE_CHECK
    assert _status() == sdpa.SDPA_OK  # cleared by the read
    got = out.cpu()
    assert torch.isnan(got[2].float()).all()
    np.testing.assert_array_equal(f64(kc[2]), f64(d["k_cache"][2]))  # skipped: cache untouched
    for b in [0, 1, 3, 5]:
        want, _, _ = oracle.sdpa_decode_with_cache(
            f64(d["q"][b:b + 1]), f64(d["k_new"][b:b + 1]), f64(d["v_new"][b:b + 1]),
            f64(d["k_cache"][b:b + 1]), f64(d["v_cache"][b:b + 1]), index[b:b + 1])
        assert_matches(got[b:b + 1], want, TOL, f"sequence {b} next to a bad index")
    # the next valid call starts from a clear status word
    rc = _call_static(q, kn, vn, kc, vc, d["index"].to(DEV), out)
    assert rc == sdpa.SDPA_OK and _status() == sdpa.SDPA_OK


def test_static_scratch_rejects_calls_that_do_not_fit_or_are_invalid():
    q = torch.empty((512, 1, 32, 128), dtype=torch.bfloat16, device=DEV)
    kc = torch.empty((512, 8192, 8, 128), dtype=torch.bfloat16, device="meta")
    p = _params(q, kc, kc)
    need = sdpa.lib.sdpa_workspace_size(ctypes.byref(p))
    assert need > 40 << 20
    rc = fn(ctypes.byref(p), q.data_ptr(), 16, 16, 16, 16, 16, q.data_ptr(), None)
    assert rc == sdpa.SDPA_ERR_WORKSPACE
    assert "static scratch" in sdpa.lib.sdpa_last_error().decode()
    # an invalid argument is refused before anything is queued (the status word is untouched)
    small = torch.empty((2, 1, 4, 128), dtype=torch.bfloat16, device=DEV)
    kc2 = torch.empty((2, 64, 1, 128), dtype=torch.bfloat16, device=DEV)
    p = _params(small, kc2, kc2)
    p.causal = sdpa.SDPA_CAUSAL_TOP_LEFT
    rc = fn(ctypes.byref(p), small.data_ptr(), 16, 16, kc2.data_ptr(), kc2.data_ptr(), 16, small.data_ptr(), None)
    assert rc == sdpa.SDPA_ERR_INVALID_ARG
