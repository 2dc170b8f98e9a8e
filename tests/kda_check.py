"""Element-wise comparison of CUDA results with the fp64 oracle.

Tolerances (written here once, used by every parity test):

* bf16 q/k/v with fp32 gates and state: |x - ref| <= 2e-3 + 1e-2 * |ref| for
  every element of ``out`` and ``S_T`` (max-abs 2e-3, relative 1e-2); final
  states (fp32 ``S_T``, state caches) are also held to a plain max-abs of 2e-3.
* fp32 q/k/v: |x - ref| <= 1e-4 for every element.

Every comparison records its margin (max-abs error, max-rel error and the
worst error / bound ratio) in ``RECORDS``; ``tests/conftest.py`` prints the
table at the end of the run, so a passing run shows how much room is left.
"""
import numpy as np
import torch

BF16_ATOL, BF16_RTOL = 2e-3, 1e-2
BF16_STATE_MAX_ABS = 2e-3
F32_ATOL, F32_RTOL = 1e-4, 0.0


def tol_for(dtype):
    return (F32_ATOL, F32_RTOL) if dtype == torch.float32 else (BF16_ATOL, BF16_RTOL)


def state_max_abs(dtype):
    """The plain max-abs bound of final states: 2e-3 for bf16 inputs (the fp32 bound is already absolute)."""
    return None if dtype == torch.float32 else BF16_STATE_MAX_ABS


RECORDS = []   # (what, max_abs, max_rel, worst error / bound)


def to_np(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def assert_close(x, ref, atol, rtol, what="", max_abs=None):
    """Every element within atol + rtol*|ref| (and, if given, within max_abs of ref);
    report max-abs / max-rel on failure."""
    x, ref = to_np(x), to_np(ref)
    assert x.shape == ref.shape, f"{what}: shape {x.shape} vs {ref.shape}"
    if x.size == 0:
        return {"max_abs": 0.0, "max_rel": 0.0}
    assert np.isfinite(x).all(), f"{what}: non-finite values in the CUDA result"
    err = np.abs(x - ref)
    bound = atol + rtol * np.abs(ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    stats = {"max_abs": float(err.max()),
             "max_rel": float((err / np.maximum(np.abs(ref), 1e-30)).max()),
             "ratio": float((err / bound).max())}
    RECORDS.append((what, stats["max_abs"], stats["max_rel"], stats["ratio"]))
    assert (err <= bound).all(), (
        f"{what}: {int((err > bound).sum())} of {err.size} elements out of tolerance "
        f"(atol {atol}, rtol {rtol}); max_abs {stats['max_abs']:.3e}, error/bound "
        f"{stats['ratio']:.3f}; worst at {worst}: "
        f"got {x[worst]:.6e}, want {ref[worst]:.6e}")
    if max_abs is not None:
        assert stats["max_abs"] <= max_abs, f"{what}: max_abs {stats['max_abs']:.3e} above {max_abs}"
    return stats
