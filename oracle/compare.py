"""Element-wise comparison of a GPU result with the float64 oracle.

TEST INFRASTRUCTURE, like the rest of this package: used by the GPU tests
and by ``__graft_entry__.smoke()``.

Tolerance per element: |gpu - oracle| <= ATOL + RTOL * |oracle|.
  * bf16 inputs, fp32 accumulation: 2e-3 / 1e-2 (the stated bound, read as
    one combined allclose: bf16 output rounding alone is up to 2^-9
    relative, so demanding both bounds at once would fail a correct kernel
    on short contexts whose outputs are of order 1).
  * fp32 inputs: 1e-5 / 1e-5 (the stated bound).
  * fp16 inputs (no bound is stated): derived from fp16's own rounding.  The
    output is rounded once to fp16, a relative error of at most 2^-11
    (4.9e-4); everything before it is fp32 arithmetic, with each softmax
    weight carried as a high and a low fp16 part (about 22 significant
    bits).  RTOL = 2e-3 is four times the output rounding; ATOL = 2e-4
    covers the fp32 arithmetic on outputs near zero.
"""
from __future__ import annotations

import numpy as np

TOL = {"bf16": (2e-3, 1e-2), "f16": (2e-4, 2e-3), "f32": (1e-5, 1e-5)}


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    atol, rtol = TOL[dtype]
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements outside tolerance; first at "
                             f"{tuple(idx)} got {got[tuple(idx)]!r} ref {ref[tuple(idx)]!r}; "
                             f"max abs {err.max():.3e}, max rel {(err / np.maximum(np.abs(ref), 1e-30)).max():.3e}")


def pool_equal(dev_pool, ref_pool: np.ndarray, dtype: str) -> bool:
    """Bitwise equality of a device pool (torch tensor) with the oracle's pool."""
    import torch
    from synth.device import to_device
    ref = to_device(ref_pool, dtype, dev_pool.device)
    iv = torch.int32 if dtype == "f32" else torch.int16
    return bool(torch.equal(dev_pool.view(iv), ref.view(iv)))
