"""pa_decode_no_alloc: the decode entry point for callers that cannot
allocate device memory (a host framework that hands the library no device
allocation, or code where cudaMalloc is not allowed).  It runs on a workspace
array built into the library.  Checked through the C ABI against pa_decode
with a caller-provided workspace and against the float64 oracle, on two calls
in a row, within the decode parity tolerance; its error word is read back
through pa_no_alloc_device_error.

Collected last on purpose, so that a run stopping at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import synth
import paged_kv_cache_472_b200 as pa
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def _no_alloc(dev, case, shape, plan, out):
    stream = torch.cuda.current_stream().cuda_stream
    return pa.lib.pa_decode_no_alloc(dev.q.data_ptr(), dev.k_cache.data_ptr(), dev.v_cache.data_ptr(),
                                     dev.block_tables.data_ptr(), dev.context_lens.data_ptr(),
                                     ctypes.c_float(case.scale), out.data_ptr(), ctypes.byref(shape),
                                     ctypes.byref(plan), stream)


@pytest.mark.parametrize("cid,batch,partition", [(2, None, 0), (4, 2, 512), (1, None, 0), (5, 48, 0)])
def test_no_alloc_matches_workspace_decode(orc, cid, batch, partition):
    case = synth.make_config(cid, batch=batch)
    # the caller-workspace entry point (after the step's append)
    dev, dec, err = H.run(case, partition, max_context_len=int(case.max_blocks_per_seq * case.block_size))
    assert err == 0
    ref_ws = H.out_f64(dev)
    kc, vc = orc.kv_append(case)
    ref = orc.decode(case, kc, vc)
    shape, plan = dec.shape, dec.plan
    assert plan.workspace_bytes <= 16 << 20
    pa.pa_no_alloc_device_error(clear=True)
    for call in range(2):   # the array keeps the previous call's contents
        out = torch.full_like(dev.out, float("nan"))
        st = _no_alloc(dev, case, shape, plan, out)
        assert st == 0, pa.pa_last_error_message()
        torch.cuda.synchronize()
        got = out.float().cpu().numpy().astype(np.float64)
        H.assert_close(got, ref_ws, case.dtype, f"no-alloc call {call} vs pa_decode")
        H.assert_close(got, ref, case.dtype, f"no-alloc call {call} vs oracle")
    assert pa.pa_no_alloc_device_error() == 0


def test_no_alloc_reports_a_bad_block_id_then_recovers(orc):
    """A block id outside the pool is flagged in the built-in array's error
    word (not lost), the word stays set until it is cleared, and the next
    good call is correct."""
    case = synth.build_case("no_alloc_badid", dtype="bf16", Hq=16, Hkv=8, D=128, block_size=16,
                            context_lens=[40, 70, 300], seed=31)
    dev, dec, err = H.run(case, 0)
    assert err == 0
    shape, plan = dec.shape, dec.plan
    pa.pa_no_alloc_device_error(clear=True)
    bad = case.block_tables.copy()
    bad[1, 2] = case.num_blocks + 5
    good_tables = dev.block_tables
    dev.block_tables = torch.from_numpy(bad).cuda()
    out = torch.full_like(dev.out, float("nan"))
    assert _no_alloc(dev, case, shape, plan, out) == 0
    torch.cuda.synchronize()
    assert pa.pa_no_alloc_device_error() & pa.DEVERR_BLOCK_ID
    dev.block_tables = good_tables
    assert _no_alloc(dev, case, shape, plan, out) == 0   # the word gathers errors until cleared
    assert pa.pa_no_alloc_device_error(clear=True) & pa.DEVERR_BLOCK_ID
    assert _no_alloc(dev, case, shape, plan, out) == 0
    assert pa.pa_no_alloc_device_error() == 0
    kc, vc = orc.kv_append(case)
    H.assert_close(out.float().cpu().numpy().astype(np.float64), orc.decode(case, kc, vc), case.dtype,
                   "no-alloc after an error")


def test_no_alloc_rejects_plans_beyond_its_array():
    # a batch of 1024 requests needs one 16.6 KB partial per request, more than 16 MiB
    s = pa.Shape(1024, 32, 8, 128, 16, 70000, 1024, pa.DTYPE_BF16)
    plan = pa.pa_plan(s, 16384, 16, 148)
    assert plan.workspace_bytes > 16 << 20
    st = pa.lib.pa_decode_no_alloc(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, ctypes.c_float(0.1), 1 << 20,
                                   ctypes.byref(s), ctypes.byref(plan), None)
    assert st == pa.PA_ERR_WORKSPACE
