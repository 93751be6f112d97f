"""Helpers shared by the GPU parity tests: element-wise comparison with the oracle.

The tolerances are max-abs 1e-5 for fp32 outputs and 1e-2 for bf16/fp16 outputs (fp32
accumulation). For a 16-bit output the bound applies to the value the kernel computes before
it stores it: the stored number is that value rounded to nearest in the output type, which by
itself moves it by up to half a unit in the last place (2^-9 relative for bf16, 2^-12 for fp16,
i.e. 0.0156 at |out| in [4, 8) in bf16). No kernel can meet a flat 1e-2 there: a causal GQA
prefill output whose float64 value is 4.0188 is stored as the bf16 number 4.03125, its correct
rounding, 0.0125 away. So a 16-bit element passes when |got - oracle| <= tol + ulp(got) / 2.
"""
import numpy as np
import torch

TOL = {torch.float32: 1e-5, torch.float16: 1e-2, torch.bfloat16: 1e-2}
_MANTISSA_BITS = {torch.bfloat16: 7, torch.float16: 10}
_MIN_EXP = {torch.bfloat16: -126, torch.float16: -14}


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def half_ulp(values: np.ndarray, dtype) -> np.ndarray:
    """Half the spacing of `dtype` numbers at each of `values` (which are numbers of that type)."""
    if dtype not in _MANTISSA_BITS:
        return np.zeros_like(values)
    a = np.abs(values)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, _MIN_EXP[dtype])
    return np.where(a > 0, np.ldexp(0.5, (e - _MANTISSA_BITS[dtype]).astype(np.int64)), 0.0)


def assert_matches(got, want, tol, what=""):
    """Max-abs error within `tol` (plus the output's own rounding for a 16-bit tensor `got`); NaN
    exactly where the oracle has NaN. Returns the largest error beyond that rounding."""
    dtype = got.dtype if isinstance(got, torch.Tensor) else None
    g, w = f64(got), f64(want)
    assert g.shape == w.shape, f"{what}: shape {g.shape} vs {w.shape}"
    gn, wn = np.isnan(g), np.isnan(w)
    assert (gn == wn).all(), f"{what}: NaN pattern differs at {np.argwhere(gn != wn)[:5].tolist()}"
    ok = ~wn
    if ok.any():
        err = np.abs(g[ok] - w[ok])
        excess = err - half_ulp(g[ok], dtype)
        i = int(np.argmax(excess))
        assert excess[i] <= tol, (f"{what}: max-abs error {err[i]:.3e} at oracle value {w[ok][i]:.4f} "
                                  f"(got {g[ok][i]:.4f}), {excess[i]:.3e} beyond the output's rounding > {tol:g}")
        return float(max(excess[i], 0.0))
    return 0.0
