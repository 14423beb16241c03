"""Shared helpers for the GPU parity tests: upload a seeded case, run the
library through its C ABI, and compare with the float64 oracle."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import synth
from paged_kv_cache_472_b200 import DTYPE_BF16, DTYPE_F16, DTYPE_F32, Shape
from paged_kv_cache_472_b200.session import PagedDecoder

# Tolerances of the decode parity check, per element:
#   |gpu - oracle| <= ATOL + RTOL * |oracle|
# bf16 inputs with fp32 accumulation: 2e-3 absolute / 1e-2 relative.  The
# bf16 output rounding alone is up to 2^-9 relative, so the two bounds are
# combined as allclose rather than required together.  fp32 inputs: 1e-5.
# fp16 inputs (no bound is stated for them): the bf16 bound, which the fp16
# output rounding (2^-11 relative) sits well inside.
TOL = {"bf16": (2e-3, 1e-2), "f16": (2e-3, 1e-2), "f32": (1e-5, 1e-5)}


def _vals(a: np.ndarray, dtype: str, device) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if dtype == "bf16":
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    if dtype == "f16":
        return torch.from_numpy(a.view(np.int16)).view(torch.float16).to(device)
    return torch.from_numpy(a).to(device)


@dataclass
class DeviceCase:
    q: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    slot_mapping: torch.Tensor
    out: torch.Tensor


def upload(case, device="cuda") -> DeviceCase:
    v = lambda a: _vals(a, case.dtype, device)
    i = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
    q = v(case.q)
    return DeviceCase(q=q, k_new=v(case.k_new), v_new=v(case.v_new), k_cache=v(case.k_cache),
                      v_cache=v(case.v_cache), block_tables=i(case.block_tables), context_lens=i(case.context_lens),
                      slot_mapping=i(case.slot_mapping), out=torch.full_like(q, float("nan")))


def shape_of(case) -> Shape:
    return Shape(case.B, case.Hq, case.Hkv, case.D, case.block_size, case.num_blocks, case.max_blocks_per_seq,
                 {"f32": DTYPE_F32, "bf16": DTYPE_BF16, "f16": DTYPE_F16}[case.dtype])


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


def pool_equal(dev_pool: torch.Tensor, ref_pool: np.ndarray, dtype: str) -> bool:
    ref = _vals(ref_pool, dtype, dev_pool.device)
    iv = torch.int32 if dtype == "f32" else torch.int16
    return bool(torch.equal(dev_pool.view(iv), ref.view(iv)))


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
