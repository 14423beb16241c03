"""pa_kv_append against the oracle's append: the whole pool, bit for bit."""
import numpy as np
import pytest
import torch

import synth
from paged_kv_cache_472_b200 import DEVERR_SLOT
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cid", [1, 2, 3, 4, 5])
def test_append_bit_exact(orc, cid):
    case = synth.make_config(cid)
    dev = H.upload(case)
    dec = H.PagedDecoder(H.shape_of(case), int(case.context_lens.max()), 0)
    dec.append(dev.k_new, dev.v_new, dev.slot_mapping, dev.k_cache, dev.v_cache)
    torch.cuda.synchronize()
    kc, vc = orc.kv_append(case)
    assert H.pool_equal(dev.k_cache, kc, case.dtype)
    assert H.pool_equal(dev.v_cache, vc, case.dtype)
    assert dec.device_error() == 0


def test_append_skips_negative_and_flags_out_of_range(orc):
    case = synth.make_config(2, batch=8)
    case.slot_mapping = case.slot_mapping.copy()
    case.slot_mapping[1] = -1
    bad = case.slot_mapping.copy()
    bad[3] = case.num_blocks * case.block_size      # one past the pool
    dev = H.upload(case)
    dev.slot_mapping = torch.from_numpy(bad).cuda()
    dec = H.PagedDecoder(H.shape_of(case), int(case.context_lens.max()), 0)
    dec.append(dev.k_new, dev.v_new, dev.slot_mapping, dev.k_cache, dev.v_cache)
    torch.cuda.synchronize()
    assert dec.device_error() & DEVERR_SLOT
    ok = case.slot_mapping.copy()
    ok[3] = -1                                       # the oracle's view: that request wrote nothing
    case.slot_mapping = ok
    kc, vc = orc.kv_append(case)
    assert H.pool_equal(dev.k_cache, kc, case.dtype)
    assert H.pool_equal(dev.v_cache, vc, case.dtype)


def test_append_fp32_and_odd_heads(orc):
    case = synth.build_case("odd", dtype="f32", Hq=6, Hkv=3, D=64, block_size=32, context_lens=[1, 32, 33, 95],
                            seed=3, pool="factor", pool_factor=2.0)
    dev = H.upload(case)
    dec = H.PagedDecoder(H.shape_of(case), 95, 0)
    dec.append(dev.k_new, dev.v_new, dev.slot_mapping, dev.k_cache, dev.v_cache)
    torch.cuda.synchronize()
    kc, vc = orc.kv_append(case)
    assert H.pool_equal(dev.k_cache, kc, "f32") and H.pool_equal(dev.v_cache, vc, "f32")
