"""Helpers shared by the GPU parity tests: element-wise comparison with the oracle."""
import numpy as np
import torch

TOL = {torch.float32: 1e-5, torch.float16: 1e-2, torch.bfloat16: 1e-2}


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def assert_matches(got, want, tol, what=""):
    """Max-abs error within `tol`; NaN exactly where the oracle has NaN."""
    g, w = f64(got), f64(want)
    assert g.shape == w.shape, f"{what}: shape {g.shape} vs {w.shape}"
    gn, wn = np.isnan(g), np.isnan(w)
    assert (gn == wn).all(), f"{what}: NaN pattern differs at {np.argwhere(gn != wn)[:5].tolist()}"
    ok = ~wn
    if ok.any():
        err = np.abs(g[ok] - w[ok])
        i = int(np.argmax(err))
        assert err[i] <= tol, (f"{what}: max-abs error {err[i]:.3e} > {tol:g} "
                               f"(oracle value there {w[ok][i]:.4f}, got {g[ok][i]:.4f})")
        return float(err[i])
    return 0.0
