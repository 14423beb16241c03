"""pa_prefill (chunked prefill over the paged cache) against the float64
oracle on the same seeded inputs: the new tokens' K/V are written with
pa_kv_append (one row per new token), then every new token attends causally
to its request's positions up to its own."""
import dataclasses

import numpy as np
import pytest
import torch

import synth
import paged_kv_cache_472_b200 as pa
from paged_kv_cache_472_b200 import DEVERR_BLOCK_ID, DEVERR_CONTEXT_LEN, Shape
from synth.device import upload_prefill
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def _dtype_code(dtype):
    return {"f32": pa.DTYPE_F32, "bf16": pa.DTYPE_BF16, "f16": pa.DTYPE_F16}[dtype]


def run_prefill(pc, dev=None, max_new=None, append=True):
    dev = dev or upload_prefill(pc)
    shape = Shape(pc.B, pc.Hq, pc.Hkv, pc.D, pc.block_size, pc.num_blocks, pc.max_blocks_per_seq,
                  _dtype_code(pc.dtype))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    if append:
        ashape = Shape(pc.T, pc.Hq, pc.Hkv, pc.D, pc.block_size, pc.num_blocks, pc.max_blocks_per_seq,
                       _dtype_code(pc.dtype))
        pa.pa_kv_append(dev["k_new"], dev["v_new"], dev["slot_mapping"], dev["k_cache"], dev["v_cache"], ashape, err)
    mx = int(pc.new_tokens().max()) if max_new is None else max_new
    plan = pa.pa_prefill_plan(shape, mx)
    pa.pa_prefill(dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"], dev["context_lens"],
                  dev["query_start"], pc.scale, dev["out"], shape, plan, err)
    torch.cuda.synchronize()
    return dev, int(err.item()), plan


def out_f64(dev):
    return dev["out"].float().cpu().numpy().astype(np.float64)


def check(orc, pc, what=""):
    dev, err, plan = run_prefill(pc)
    assert err == 0, f"device error word {err:#x}"
    H.assert_close(out_f64(dev), orc.prefill(pc), pc.dtype, what or pc.name)
    return dev


@pytest.mark.parametrize("pid,batch,chunk", [(1, 2, 96), (1, 3, 200), (2, 4, 130)])
def test_prefill_workloads_full_output(orc, pid, batch, chunk):
    check(orc, synth.make_prefill_config(pid, batch=batch, chunk=chunk))


@pytest.mark.parametrize("pid", [1, 2])
def test_prefill_workloads_full_size_full_output(orc, pid):
    """Every output row of both prefill workloads at full size against the
    oracle, launched as bench.py --prefill times it (the append of every new
    token, then one pa_prefill launch planned for the longest chunk)."""
    pc = synth.make_prefill_config(pid)
    dev, err, plan = run_prefill(pc)
    assert err == 0
    H.assert_close(out_f64(dev), orc.prefill(pc), pc.dtype, pc.name + " full size")


EDGE = [
    # name, dtype, Hq, Hkv, D, bs, context_lens, new_tokens
    ("fresh_mha", "bf16", 4, 4, 64, 16, [40, 17, 1], [40, 17, 1]),
    ("one_token_each", "bf16", 16, 8, 128, 16, [300, 17, 64], [1, 1, 1]),
    ("gqa8_long_history", "bf16", 32, 4, 128, 16, [2000, 129], [70, 129]),
    ("mqa_g32_bs256", "bf16", 32, 1, 128, 256, [1000, 300], [300, 7]),
    ("g2_bs64", "bf16", 8, 4, 64, 64, [257, 63, 64], [200, 63, 1]),
    ("fp16", "f16", 16, 8, 128, 16, [500, 33], [120, 33]),
    ("ragged_tail_tiles", "bf16", 8, 2, 128, 32, [65, 129, 191], [65, 65, 66]),
    ("g64_bs128", "bf16", 64, 1, 64, 128, [700, 129, 5], [50, 129, 5]),
    ("g128_one_token_tiles", "f16", 128, 1, 128, 16, [300, 40], [9, 40]),
]


@pytest.mark.parametrize("name,dtype,Hq,Hkv,D,bs,lens,new", EDGE)
def test_prefill_edge_shapes(orc, name, dtype, Hq, Hkv, D, bs, lens, new):
    pc = synth.build_prefill_case(name, dtype=dtype, Hq=Hq, Hkv=Hkv, D=D, block_size=bs, context_lens=lens,
                                  new_tokens=new, seed=sum(lens) + 7, pool="factor", pool_factor=1.5)
    check(orc, pc, name)


def test_prefill_more_pairs_than_ranked(orc):
    """More (request, CTA tile) pairs than the kernel ranks in shared memory
    (1100 requests x 2 tiles): the CTAs fall back to taking the pairs in
    request order, every row still against the oracle."""
    rng = np.random.default_rng(5)
    B = 1100
    new = rng.integers(1, 4, size=B)
    new[7] = 200  # one long chunk: two CTA tiles of 2 x 64 tokens per request
    lens = new + rng.integers(0, 40, size=B)
    pc = synth.build_prefill_case("many_pairs", dtype="bf16", Hq=4, Hkv=2, D=64, block_size=16,
                                  context_lens=lens.tolist(), new_tokens=new.tolist(), seed=23, pool="factor",
                                  pool_factor=1.25)
    dev, err, plan = run_prefill(pc)
    assert pc.B * plan.num_qtiles > 2048
    assert err == 0, f"device error word {err:#x}"
    H.assert_close(out_f64(dev), orc.prefill(pc), pc.dtype, pc.name)


@pytest.mark.parametrize("scale", [-0.2, 0.0, 0.5])
def test_prefill_any_scale(orc, scale):
    """A negative scale (the kernel feeds q negated and uses |scale|), zero
    (uniform weights over each row's visible keys) and a large one (peaked
    rows, where the low part of each weight matters)."""
    base = synth.build_prefill_case("scale", dtype="bf16", Hq=16, Hkv=4, D=128, block_size=16,
                                    context_lens=[300, 40], new_tokens=[150, 40], seed=11, pool="factor",
                                    pool_factor=1.5)
    check(orc, dataclasses.replace(base, scale=scale, name=f"scale {scale}"), f"scale {scale}")


def test_prefill_one_new_token_matches_decode(orc):
    """One new token per request: prefill and decode give the same rows (both
    against the oracle)."""
    dc = synth.make_config(2, batch=5)
    pc = synth.PagedPrefillCase(
        name="decode-as-prefill", dtype=dc.dtype, B=dc.B, T=dc.B, Hq=dc.Hq, Hkv=dc.Hkv, D=dc.D,
        block_size=dc.block_size, num_blocks=dc.num_blocks, max_blocks_per_seq=dc.max_blocks_per_seq,
        context_lens=dc.context_lens, query_start=np.arange(dc.B + 1, dtype=np.int32),
        block_tables=dc.block_tables, slot_mapping=dc.slot_mapping, q=dc.q, k_new=dc.k_new, v_new=dc.v_new,
        k_cache=dc.k_cache, v_cache=dc.v_cache, scale=dc.scale)
    dev = check(orc, pc, "one token")
    ddev, _, derr = H.run(dc, 0)
    assert derr == 0
    H.assert_close(out_f64(dev), orc.decode(dc), dc.dtype, "prefill vs decode oracle")
    H.assert_close(H.out_f64(ddev), orc.prefill(pc), dc.dtype, "decode vs prefill oracle")


def test_prefill_bad_inputs_are_flagged_not_faulted():
    pc = synth.build_prefill_case("bad", dtype="bf16", Hq=8, Hkv=2, D=64, block_size=16, context_lens=[50, 40],
                                  new_tokens=[20, 10], seed=5)
    dev = upload_prefill(pc)
    dev["block_tables"][1, 0] = pc.num_blocks + 3           # a block id past the pool
    _, err, _ = run_prefill(pc, dev=dev)
    assert err & DEVERR_BLOCK_ID
    dev = upload_prefill(pc)
    dev["context_lens"][0] = 10                             # request 0: 20 new tokens, length 10
    out_before = dev["out"].clone()
    _, err, _ = run_prefill(pc, dev=dev, append=False)
    assert err & DEVERR_CONTEXT_LEN
    q0, q1 = int(pc.query_start[0]), int(pc.query_start[1])
    assert torch.equal(dev["out"][q0:q1].isnan(), out_before[q0:q1].isnan())   # its rows are left alone
    assert not dev["out"][q1:].isnan().any()                                    # the other request ran

