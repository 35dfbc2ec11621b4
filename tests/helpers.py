"""Shared test helpers: the error metric and tensor conversions (no operator arithmetic)."""
import numpy as np
import torch

TOL_BF16 = 2e-2   # bf16 inputs, fp32 accumulation
TOL_F32 = 1e-4    # fp32 path


def f64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def rel_err(x, ref):
    """max_i |x_i - r_i| / max(|r_i|, rms(r)): per-element relative error floored at the RMS."""
    x, ref = f64(x), f64(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    rms = np.sqrt(np.mean(ref * ref))
    if rms == 0:
        return float(np.max(np.abs(x - ref)))
    den = np.maximum(np.abs(ref), rms)
    return float(np.max(np.abs(x - ref) / den))


def tol_for(dtype):
    return TOL_F32 if dtype == torch.float32 else TOL_BF16


def assert_close(name, x, ref, tol):
    e = rel_err(x, ref)
    assert np.all(np.isfinite(f64(x))), f"{name}: non-finite values"
    assert e <= tol, f"{name}: rel err {e:.3e} > {tol:.1e}"
    return e


def cuda(d):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
