"""pa_decode_no_alloc: the decode entry point for callers that cannot
allocate device memory (it runs on a workspace array built into the
library).  Checked through the C ABI against pa_decode with a caller-provided
workspace, on two calls in a row, within the decode parity tolerance.

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


@pytest.mark.parametrize("cid,batch,partition", [(2, None, 0), (4, 2, 512), (1, None, 0)])
def test_no_alloc_matches_workspace_decode(cid, batch, partition):
    case = synth.make_config(cid, batch=batch)
    # reference: the caller-workspace entry point (after the step's append)
    dev, dec, err = H.run(case, partition, max_context_len=int(case.max_blocks_per_seq * case.block_size))
    assert err == 0
    ref = H.out_f64(dev)
    shape, plan = dec.shape, dec.plan
    assert plan.workspace_bytes <= 16 << 20
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):   # the array keeps the previous call's contents
        out = torch.full_like(dev.out, float("nan"))
        st = pa.lib.pa_decode_no_alloc(dev.q.data_ptr(), dev.k_cache.data_ptr(), dev.v_cache.data_ptr(),
                                       dev.block_tables.data_ptr(), dev.context_lens.data_ptr(),
                                       ctypes.c_float(case.scale), out.data_ptr(), ctypes.byref(shape),
                                       ctypes.byref(plan), stream)
        assert st == 0, pa.pa_last_error_message()
        torch.cuda.synchronize()
        got = out.float().cpu().numpy().astype(np.float64)
        H.assert_close(got, ref, case.dtype, f"no-alloc call {call}")


def test_no_alloc_rejects_plans_beyond_its_array():
    # a batch of 1024 requests needs one 16.6 KB partial per request, more than 16 MiB
    s = pa.Shape(1024, 32, 8, 128, 16, 70000, 1024, pa.DTYPE_BF16)
    plan = pa.pa_plan(s, 16384, 16, 148)
    assert plan.workspace_bytes > 16 << 20
    st = pa.lib.pa_decode_no_alloc(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, ctypes.c_float(0.1), 1 << 20,
                                   ctypes.byref(s), ctypes.byref(plan), None)
    assert st == pa.PA_ERR_WORKSPACE
