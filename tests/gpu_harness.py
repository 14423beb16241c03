"""Shared helpers for the GPU parity tests: upload a seeded case, run the
library through its C ABI, and compare with the float64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import synth
from paged_kv_cache_472_b200 import Shape
from paged_kv_cache_472_b200.session import PagedDecoder

from oracle.compare import TOL, assert_close, pool_equal  # noqa: F401  (re-exported for the tests)
from synth.device import DeviceCase, shape_fields, to_device as _vals, upload  # noqa: F401


def shape_of(case) -> Shape:
    return Shape(*shape_fields(case))


def run(case, partition_tokens: int = 0, max_context_len: int | None = None, dev: DeviceCase | None = None,
        append: bool = True, num_sms: int = 0, flags: int = 0):
    """Append then decode on the GPU; returns (device case, decoder, device error word).
    `flags`: pa_plan_t.flags for the decode."""
    dev = dev or upload(case)
    mc = max_context_len if max_context_len is not None else max(int(case.context_lens.max()), 1)
    dec = PagedDecoder(shape_of(case), mc, partition_tokens, num_sms)
    dec.plan.flags = flags
    if append:
        dec.append(dev.k_new, dev.v_new, dev.slot_mapping, dev.k_cache, dev.v_cache)
    dec.decode(dev.q, dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens, case.scale, dev.out)
    torch.cuda.synchronize()
    err = dec.device_error()
    return dev, dec, err


def out_f64(dev: DeviceCase) -> np.ndarray:
    return dev.out.float().cpu().numpy().astype(np.float64)


def sample_pairs(case, n: int, seed: int = 0) -> np.ndarray:
    """(request, head) pairs: the longest and the shortest request (all
    heads) plus n random pairs."""
    rng = np.random.default_rng(seed)
    lens = case.context_lens
    pairs = {(int(np.argmax(lens)), h) for h in range(case.Hq)}
    pairs |= {(int(np.argmin(lens)), h) for h in range(case.Hq)}
    target = min(2 * case.Hq + n, case.B * case.Hq)
    while len(pairs) < target:
        pairs.add((int(rng.integers(case.B)), int(rng.integers(case.Hq))))
    return np.array(sorted(pairs), dtype=np.int32)
