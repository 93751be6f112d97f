"""The decode entry point for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc (a plug-in inside a framework that owns all
device memory, or a decode loop that must not touch the allocator mid-run), so they cannot pass
the workspace sdpa_decode_with_cache needs. sdpa_decode_with_cache_static takes the same
arguments minus the workspace and keeps its scratch in a fixed array inside the library. This
test calls it through the C ABI and checks it against sdpa_decode_with_cache on the same inputs,
on two calls in a row (the array keeps the previous call's contents), and checks that a call too
large for the array is refused before anything runs.
"""
import ctypes

import numpy as np
import pytest
import torch

import sdpa_inputs as si

pytestmark = pytest.mark.gpu

sdpa = pytest.importorskip("head_scaled_dot_sdpa_b200")
DEV = "cuda"
TOL = 1e-2  # bf16 outputs, as in the other decode parity tests

fn = sdpa.lib.sdpa_decode_with_cache_static
fn.argtypes = [ctypes.POINTER(sdpa.Params)] + [ctypes.c_void_p] * 8
fn.restype = ctypes.c_int


def _inputs():
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


def test_static_scratch_matches_workspace_entry_point():
    d = _inputs()
    q, kn, vn = d["q"].to(DEV), d["k_new"].to(DEV), d["v_new"].to(DEV)
    idx = d["index"].to(DEV)
    kc_ref, vc_ref = d["k_cache"].to(DEV), d["v_cache"].to(DEV)
    ref = sdpa.sdpa_decode_with_cache(q, kn, vn, kc_ref, vc_ref, idx)
    torch.cuda.synchronize()
    assert sdpa.read_device_status() == sdpa.SDPA_OK
    kc, vc = d["k_cache"].to(DEV), d["v_cache"].to(DEV)
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        rc = _call_static(q, kn, vn, kc, vc, idx, out)
        assert rc == sdpa.SDPA_OK, sdpa.lib.sdpa_last_error().decode()
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= TOL, f"call {call}: max-abs difference {err}"
        assert torch.equal(kc, kc_ref) and torch.equal(vc, vc_ref)


def test_static_scratch_rejects_calls_that_do_not_fit():
    q = torch.empty((512, 1, 32, 128), dtype=torch.bfloat16, device=DEV)
    kc = torch.empty((512, 8192, 8, 128), dtype=torch.bfloat16, device="meta")
    p = _params(q, kc, kc)
    need = sdpa.lib.sdpa_workspace_size(ctypes.byref(p))
    assert need > 32 << 20
    rc = fn(ctypes.byref(p), q.data_ptr(), 16, 16, 16, 16, 16, q.data_ptr(), None)
    assert rc == sdpa.SDPA_ERR_WORKSPACE
    assert "static scratch" in sdpa.lib.sdpa_last_error().decode()
