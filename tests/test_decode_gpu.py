"""pa_decode against the float64 oracle on the same seeded inputs.

Full outputs at sizes the oracle finishes in seconds (several tiles, ragged
tails, every split mode), and every output element at the full sizes of the
five workloads, in the launch configuration the benchmark times (one fused
append + decode launch, one CTA per SM)."""
import dataclasses
import zlib

import numpy as np
import pytest
import torch

import synth
import paged_kv_cache_472_b200 as pa
from paged_kv_cache_472_b200 import (DEVERR_BLOCK_ID, DEVERR_CONTEXT_LEN, DEVERR_SLOT, DEVERR_TIMEOUT,
                                     PLAN_NO_SPECULATION, PLAN_TEST_MISGUESS, PLAN_TEST_STALL)
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


_REF = {}


def oracle_out(orc, case):
    key = (case.name, case.seed, case.scale)
    if key not in _REF:
        _REF[key] = orc.decode(case)
    return _REF[key]


def check_full(orc, case, partition_tokens=0, what=""):
    dev, dec, err = H.run(case, partition_tokens)
    assert err == 0, f"device error word {err:#x}"
    ref = oracle_out(orc, case)
    H.assert_close(H.out_f64(dev), ref, case.dtype, what or case.name)
    return dev


# ---- the five workloads, full outputs (smaller batches where the oracle needs it) ----
@pytest.mark.parametrize("cid,batch", [(1, None), (2, None), (3, 32), (4, 2), (5, 48)])
@pytest.mark.parametrize("partition", ["balanced", "fixed", "none"])
def test_workloads_full_output(orc, cid, batch, partition):
    case = synth.make_config(cid, batch=batch)
    pt = {"balanced": 0, "fixed": case.partition_tokens or 256,
          "none": int(case.max_blocks_per_seq * case.block_size)}[partition]
    check_full(orc, case, pt, f"{case.name}/{partition}")


# ---- full sizes, every output element, launch configuration of the benchmark ----
def bench_step(case, partition_tokens, flags=0):
    """One fused append + decode launch as bench.py times it: the plan for the
    table's full capacity and the given split."""
    dev = H.upload(case)
    dec = H.PagedDecoder(H.shape_of(case), int(case.max_blocks_per_seq * case.block_size), partition_tokens)
    dec.plan.flags = flags
    dec.append_decode(dev.k_new, dev.v_new, dev.slot_mapping, dev.q, dev.k_cache, dev.v_cache, dev.block_tables,
                      dev.context_lens, case.scale, dev.out)
    torch.cuda.synchronize()
    return dev, dec


@pytest.mark.parametrize("cid", [1, 2, 3, 4, 5])
def test_workloads_full_size_full_output(orc, cid):
    """All B x Hq x D outputs of each workload at its full size against the
    oracle, and the whole pool after the append bit for bit."""
    case = synth.make_config(cid)
    dev, dec = bench_step(case, case.partition_tokens)
    assert dec.device_error() == 0
    kc, vc = orc.kv_append(case)
    assert H.pool_equal(dev.k_cache, kc, case.dtype) and H.pool_equal(dev.v_cache, vc, case.dtype)
    ref = oracle_out(orc, case)
    H.assert_close(H.out_f64(dev), ref, case.dtype, f"{case.name} full size")
    if case.partition_tokens:   # the balanced split on the same inputs, too
        dev2, dec2 = bench_step(case, 0)
        assert dec2.device_error() == 0
        H.assert_close(H.out_f64(dev2), ref, case.dtype, f"{case.name} full size balanced")


def test_split_equals_unsplit(orc):
    """Balanced, fixed and unsplit launches agree with each other (and the oracle)."""
    case = synth.make_config(4, batch=2)
    outs = []
    for pt in (0, 512, 2048, int(case.max_blocks_per_seq * case.block_size)):
        dev, _, err = H.run(case, pt)
        assert err == 0
        outs.append(H.out_f64(dev))
    for o in outs[1:]:
        H.assert_close(o, outs[0], case.dtype, "split vs split")


# ---- edge shapes ----
EDGE = [
    # name, dtype, Hq, Hkv, D, bs, lens
    ("len1", "bf16", 16, 8, 128, 16, [1, 1, 2, 1]),
    ("exact_blocks", "bf16", 32, 8, 64, 16, [16, 32, 48, 256]),
    ("block_pm1", "bf16", 16, 8, 128, 16, [15, 17, 31, 33, 47, 49]),
    ("mha8", "bf16", 8, 8, 128, 16, [5, 100, 300]),
    ("mha32_headgroups", "bf16", 32, 32, 128, 16, [40, 333, 17]),
    ("mha16_d64_two_units", "bf16", 16, 16, 64, 16, [77, 250, 1]),
    ("gqa4_d64_hkv16", "bf16", 64, 16, 64, 32, [300, 65, 2]),
    ("mqa8", "bf16", 8, 1, 128, 16, [1000, 3, 129]),
    ("mqa4_tsplit", "bf16", 4, 1, 128, 64, [700, 64, 65]),
    ("mqa32", "bf16", 32, 1, 128, 256, [3000, 257, 1]),
    ("mqa64", "bf16", 64, 1, 64, 128, [1500, 130]),
    ("gqa16", "bf16", 32, 2, 128, 32, [900, 31, 2]),
    ("tiny_heads", "bf16", 2, 2, 64, 16, [50, 3]),
    ("one_head", "f32", 1, 1, 64, 16, [33, 80]),
    ("f32_gqa4", "f32", 16, 4, 128, 32, [129, 500, 31]),
    ("f32_d64_bs256", "f32", 8, 2, 64, 256, [600, 256, 257]),
    ("bs128_d128", "bf16", 16, 8, 128, 128, [129, 1024, 383]),
    ("single_request", "bf16", 16, 8, 128, 16, [4000]),
    ("f16_gqa2", "f16", 16, 8, 128, 16, [300, 17, 1, 1100]),
    ("f16_d64_gqa4", "f16", 32, 8, 64, 32, [513, 64, 2]),
    ("f16_mqa32", "f16", 32, 1, 128, 256, [2000, 255]),
    # the tcgen05 engine (D = 128, 16 / 32 / 64 query heads per KV head): ragged tiles of 128 tokens
    ("tc_g64", "bf16", 64, 1, 128, 16, [700, 129, 1, 128]),
    ("tc_g16_ragged", "bf16", 64, 4, 128, 16, [1, 15, 16, 17, 127, 128, 129, 255, 257]),
    ("tc_g32_f16_bs64", "f16", 64, 2, 128, 64, [1000, 2, 385]),
    ("tc_g16_f16_bs256", "f16", 16, 1, 128, 256, [5000, 300, 17]),
]


@pytest.mark.parametrize("name,dtype,Hq,Hkv,D,bs,lens", EDGE, ids=[e[0] for e in EDGE])
@pytest.mark.parametrize("pt", [0, 64, 256])
def test_edge_shapes(orc, name, dtype, Hq, Hkv, D, bs, lens, pt):
    case = synth.build_case(name, dtype=dtype, Hq=Hq, Hkv=Hkv, D=D, block_size=bs, context_lens=lens,
                            seed=zlib.crc32(name.encode()) % 100000, pool="factor", pool_factor=1.25)
    check_full(orc, case, pt, f"{name}/pt{pt}")


def test_many_short_requests(orc):
    """More requests than CTAs; many requests inside one CTA's range."""
    rng = np.random.default_rng(9)
    lens = rng.integers(1, 40, size=700)
    case = synth.build_case("many_short", dtype="bf16", Hq=16, Hkv=8, D=128, block_size=16, context_lens=lens,
                            seed=9)
    check_full(orc, case, 0)


def test_fewer_tiles_than_ctas(orc):
    case = synth.build_case("few", dtype="bf16", Hq=16, Hkv=8, D=128, block_size=16, context_lens=[20, 3],
                            seed=10)
    check_full(orc, case, 0)


def test_zero_length_requests_give_zero(orc):
    case = synth.build_case("zeros", dtype="bf16", Hq=16, Hkv=8, D=128, block_size=16, context_lens=[50, 1, 70],
                            seed=11)
    dev = H.upload(case)
    lens = case.context_lens.copy()
    lens[1] = 0
    dev.context_lens = torch.from_numpy(lens).cuda()
    dev, dec, err = H.run(case, 0, dev=dev, append=False)
    assert err == 0
    got = H.out_f64(dev)
    assert np.all(got[1] == 0.0)
    ref = orc.decode(case, case.k_cache, case.v_cache, context_lens=lens)
    H.assert_close(got, ref, "bf16", "zeros")


def test_bad_block_id_is_flagged_not_faulted():
    case = synth.build_case("badid", dtype="bf16", Hq=16, Hkv=8, D=128, block_size=16, context_lens=[40, 70],
                            seed=12)
    dev = H.upload(case)
    tables = case.block_tables.copy()
    tables[1, 2] = case.num_blocks + 5          # outside the pool
    dev.block_tables = torch.from_numpy(tables).cuda()
    dev, dec, err = H.run(case, 0, dev=dev)
    assert err & DEVERR_BLOCK_ID
    torch.cuda.synchronize()                      # the context is still usable


def test_context_longer_than_table_is_flagged():
    case = synth.build_case("badlen", dtype="bf16", Hq=16, Hkv=8, D=128, block_size=16, context_lens=[40, 70],
                            seed=13, max_blocks_per_seq=5)
    dev = H.upload(case)
    lens = case.context_lens.copy()
    lens[1] = 5 * 16 + 7
    dev.context_lens = torch.from_numpy(lens).cuda()
    dev, dec, err = H.run(case, 0, dev=dev, max_context_len=80)
    assert err & DEVERR_CONTEXT_LEN


@pytest.mark.parametrize("cid,batch,pt", [(2, 8, 0), (4, 2, 512)])
def test_bounded_wait_gives_up_and_the_context_survives(orc, cid, batch, pt):
    """Failure detection on the device: with PA_PLAN_TEST_STALL the first CTA
    never receives the tiles of its first piece.  Its consumers' bounded wait
    gives up (about 2 s), PA_DEVERR_TIMEOUT is recorded, the call returns and
    the CUDA context stays usable: after pa_workspace_init the same decoder
    gives the oracle's result.  Both consumer designs: warp-level tiles
    (Qwen3-0.6B shape) and the tcgen05 engine (long-context MQA), which also
    frees its tensor memory on the way out."""
    import time
    case = synth.make_config(cid, batch=batch)
    dev, dec, err = H.run(case, pt, flags=PLAN_TEST_STALL)
    assert err & DEVERR_TIMEOUT, f"device error word {err:#x}"
    t0 = time.time()
    torch.cuda.synchronize()                       # nothing is left running
    assert time.time() - t0 < 1.0
    dec.plan.flags = 0
    pa.pa_workspace_init(dec.workspace, dec.workspace.numel())
    dev.out.fill_(float("nan"))
    dec.decode(dev.q, dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens, case.scale, dev.out)
    torch.cuda.synchronize()
    assert dec.device_error() == 0
    H.assert_close(H.out_f64(dev), oracle_out(orc, case), case.dtype, "after a timeout")


def test_repeated_calls_reuse_workspace(orc):
    """The merge counters return to zero: the same workspace serves call after call."""
    case = synth.make_config(2, batch=8)
    dev, dec, err = H.run(case, 0)
    first = dev.out.clone()
    for _ in range(3):
        dev.out.fill_(float("nan"))
        dec.decode(dev.q, dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens, case.scale, dev.out)
    torch.cuda.synchronize()
    assert torch.equal(first, dev.out)
    assert dec.device_error() == 0
    counters = dec.workspace[256:256 + 4 * case.B * case.Hkv].view(torch.int32)
    assert int(counters.abs().sum()) == 0
    header = dec.workspace[:256].view(torch.int32)   # error word, dynamic-list counters
    assert int(header.abs().sum()) == 0


def test_dynamic_grains_match_static_split(orc):
    """The same batch with a quarter of every request's tiles handed out at run
    time and with a purely static split: both match the oracle, and repeated
    calls (different CTAs taking different grains) are bit-identical."""
    case = synth.make_config(2)
    ref = oracle_out(orc, case)
    outs = []
    for share in (64, 0):
        dev = H.upload(case)
        dec = H.PagedDecoder(H.shape_of(case), int(case.context_lens.max()), 0)
        assert dec.plan.dynamic_share == 0
        dec.plan.dynamic_share = share
        dec.append(dev.k_new, dev.v_new, dev.slot_mapping, dev.k_cache, dev.v_cache)
        first = None
        for _ in range(4):
            dev.out.fill_(float("nan"))
            dec.decode(dev.q, dev.k_cache, dev.v_cache, dev.block_tables, dev.context_lens, case.scale, dev.out)
            torch.cuda.synchronize()
            if first is None:
                first = dev.out.clone()
            assert torch.equal(first, dev.out)
        assert dec.device_error() == 0
        assert int(dec.workspace[:256].view(torch.int32).abs().sum()) == 0
        H.assert_close(H.out_f64(dev), ref, case.dtype, f"dynamic share {share}")
        outs.append(H.out_f64(dev))


def test_fp16_workload_shape(orc):
    """The Qwen3-0.6B-shaped batch with fp16 values instead of bf16."""
    rng = np.random.default_rng(2002)
    lens = rng.integers(128, 2048, size=32, endpoint=True)
    case = synth.build_case("qwen3-0.6b-fp16", dtype="f16", Hq=16, Hkv=8, D=128, block_size=16,
                            context_lens=lens, seed=2002)
    check_full(orc, case, 0)


@pytest.mark.parametrize("scale", [-0.2, 0.0, 0.5])
@pytest.mark.parametrize("cid,batch", [(2, 6), (4, 2)])
def test_any_scale(orc, scale, cid, batch):
    """Negative, zero and large scales (the balanced split, with the merge)."""
    case = dataclasses.replace(synth.make_config(cid, batch=batch), scale=scale)
    check_full(orc, case, 0, f"{case.name} scale {scale}")


@pytest.mark.parametrize("cid,batch", [(2, None), (3, 32), (5, 48), (1, None)])
def test_fused_append_decode_matches_separate_calls(orc, cid, batch):
    """pa_kv_append_decode (one launch: the new token is written to its slot
    and patched into the staged tile) gives bit-identical results to the two
    separate calls."""
    case = synth.make_config(cid, batch=batch)
    dev_a, dec_a, err_a = H.run(case, 0)
    dev_b = H.upload(case)
    dec_b = H.PagedDecoder(H.shape_of(case), int(case.context_lens.max()), 0)
    for _ in range(3):   # repeated steps: the append is idempotent, the result must not change
        dec_b.append_decode(dev_b.k_new, dev_b.v_new, dev_b.slot_mapping, dev_b.q, dev_b.k_cache, dev_b.v_cache,
                            dev_b.block_tables, dev_b.context_lens, case.scale, dev_b.out)
    torch.cuda.synchronize()
    assert err_a == 0 and dec_b.device_error() == 0
    assert torch.equal(dev_a.k_cache, dev_b.k_cache) and torch.equal(dev_a.v_cache, dev_b.v_cache)
    assert torch.equal(dev_a.out, dev_b.out)
    H.assert_close(H.out_f64(dev_b), oracle_out(orc, case), case.dtype, "fused")


# ---- the early (speculative) plan: off, and always wrong (the start-over path) ----
@pytest.mark.parametrize("flags", [PLAN_NO_SPECULATION, PLAN_TEST_MISGUESS])
@pytest.mark.parametrize("cid,batch,pt", [(1, None, 0), (2, None, 0), (3, 32, 0), (4, 2, 512), (5, 48, 0)])
def test_speculation_off_and_misguessed(orc, flags, cid, batch, pt):
    """With the early plan turned off, or with every early guess made wrong on
    purpose (so each CTA plans again after the grid-dependency wait), the
    output still matches the oracle and nothing is flagged."""
    case = synth.make_config(cid, batch=batch)
    dev, dec, err = H.run(case, pt, flags=flags)
    assert err == 0, f"device error word {err:#x}"
    H.assert_close(H.out_f64(dev), oracle_out(orc, case), case.dtype, f"{case.name} flags={flags}")


@pytest.mark.parametrize("cid,batch", [(2, None), (5, 48)])
def test_fused_step_misguessed_matches(orc, cid, batch):
    """The fused step with every early guess wrong: bit-identical to the fused
    step that guessed right, over repeated steps on one workspace."""
    case = synth.make_config(cid, batch=batch)
    outs = []
    for flags in (0, PLAN_TEST_MISGUESS):
        dev = H.upload(case)
        dec = H.PagedDecoder(H.shape_of(case), int(case.context_lens.max()), 0)
        dec.plan.flags = flags
        for _ in range(3):
            dec.append_decode(dev.k_new, dev.v_new, dev.slot_mapping, dev.q, dev.k_cache, dev.v_cache,
                              dev.block_tables, dev.context_lens, case.scale, dev.out)
        torch.cuda.synchronize()
        assert dec.device_error() == 0
        outs.append(dev)
    assert torch.equal(outs[0].out, outs[1].out)
    assert torch.equal(outs[0].k_cache, outs[1].k_cache) and torch.equal(outs[0].v_cache, outs[1].v_cache)
    H.assert_close(H.out_f64(outs[1]), oracle_out(orc, case), case.dtype, "fused misguessed")


def _free_slot(case) -> int:
    used = set(int(x) for x in case.block_tables.ravel() if x >= 0)
    free = [b for b in range(case.num_blocks) if b not in used]
    assert free, "the pool has no unused block"
    return free[0] * case.block_size + 3


def test_fused_step_flags_a_slot_that_is_not_the_last_position(orc):
    """A new token sent to another slot than its request's last position: the
    fused step still writes it there, decodes from the cache as it stands and
    reports PA_DEVERR_SLOT (its contract); nothing faults."""
    base = synth.build_case("foreign_slot", dtype="bf16", Hq=16, Hkv=8, D=128, block_size=16,
                            context_lens=[300, 41, 900], seed=21, pool="factor", pool_factor=1.5)
    sm = base.slot_mapping.copy()
    sm[1] = _free_slot(base)
    case = dataclasses.replace(base, slot_mapping=sm)
    dev = H.upload(case)
    dec = H.PagedDecoder(H.shape_of(case), int(case.context_lens.max()), 0)
    dec.append_decode(dev.k_new, dev.v_new, dev.slot_mapping, dev.q, dev.k_cache, dev.v_cache, dev.block_tables,
                      dev.context_lens, case.scale, dev.out)
    torch.cuda.synchronize()
    assert dec.device_error() & DEVERR_SLOT
    kc, vc = orc.kv_append(case)
    assert H.pool_equal(dev.k_cache, kc, case.dtype) and H.pool_equal(dev.v_cache, vc, case.dtype)
    H.assert_close(H.out_f64(dev), orc.decode(case, kc, vc), case.dtype, "foreign slot")


def test_fused_step_appends_for_zero_length_requests(orc):
    """context_lens[b] = 0 with a slot: out[b] = 0 and the token still lands."""
    base = synth.build_case("zero_append", dtype="bf16", Hq=16, Hkv=8, D=128, block_size=16,
                            context_lens=[70, 1, 200], seed=22, pool="factor", pool_factor=1.5)
    lens = base.context_lens.copy()
    lens[1] = 0
    sm = base.slot_mapping.copy()
    sm[1] = _free_slot(base)
    case = dataclasses.replace(base, context_lens=lens, slot_mapping=sm)
    dev = H.upload(case)
    dec = H.PagedDecoder(H.shape_of(case), 200, 0)
    dec.append_decode(dev.k_new, dev.v_new, dev.slot_mapping, dev.q, dev.k_cache, dev.v_cache, dev.block_tables,
                      dev.context_lens, case.scale, dev.out)
    torch.cuda.synchronize()
    assert dec.device_error() == 0
    kc, vc = orc.kv_append(case)
    assert H.pool_equal(dev.k_cache, kc, case.dtype) and H.pool_equal(dev.v_cache, vc, case.dtype)
    got = H.out_f64(dev)
    assert np.all(got[1] == 0.0)
    H.assert_close(got, orc.decode(case, kc, vc), case.dtype, "zero-length append")


@pytest.mark.parametrize("name,dtype,Hq,Hkv,D,bs,lens,pt", [
    ("fused_f32", "f32", 16, 4, 128, 32, [129, 500, 31, 1], 0),
    ("fused_mqa32", "bf16", 32, 1, 128, 256, [3000, 257, 1], 0),
    ("fused_tsplit", "bf16", 4, 1, 128, 64, [700, 64, 65], 0),
    ("fused_fixed", "bf16", 16, 8, 128, 16, [1000, 17, 513], 256),
    ("fused_f16_d64", "f16", 32, 8, 64, 32, [513, 64, 2], 0),
])
def test_fused_step_edge_shapes(orc, name, dtype, Hq, Hkv, D, bs, lens, pt):
    """The fused step on engines, layouts and splits the workloads do not reach."""
    case = synth.build_case(name, dtype=dtype, Hq=Hq, Hkv=Hkv, D=D, block_size=bs, context_lens=lens,
                            seed=zlib.crc32(name.encode()) % 100000, pool="factor", pool_factor=1.25)
    dev = H.upload(case)
    dec = H.PagedDecoder(H.shape_of(case), int(max(lens)), pt)
    dec.append_decode(dev.k_new, dev.v_new, dev.slot_mapping, dev.q, dev.k_cache, dev.v_cache, dev.block_tables,
                      dev.context_lens, case.scale, dev.out)
    torch.cuda.synchronize()
    assert dec.device_error() == 0
    kc, vc = orc.kv_append(case)
    assert H.pool_equal(dev.k_cache, kc, case.dtype) and H.pool_equal(dev.v_cache, vc, case.dtype)
    H.assert_close(H.out_f64(dev), oracle_out(orc, case), case.dtype, name)


def test_step_staging_one_copy_matches(orc):
    """Inputs staged in one pinned buffer and uploaded with one copy (the
    end-to-end path of the benchmark) give the same bytes as separate device
    tensors."""
    from paged_kv_cache_472_b200.session import StepStaging
    case = synth.make_config(2, batch=6)
    dev = H.upload(case)
    names = StepStaging.ORDER
    stg = StepStaging({n: (tuple(getattr(dev, n).shape), getattr(dev, n).dtype) for n in names},
                      tuple(dev.out.shape), dev.out.dtype)
    for n in names:
        stg.host[n].copy_(getattr(dev, n).cpu())
        assert stg.dev[n].data_ptr() % 256 == 0
    stg.upload()
    ref = H.upload(case)
    dec = H.PagedDecoder(H.shape_of(case), int(case.context_lens.max()), 0)
    dec.append_decode(stg.dev["k_new"], stg.dev["v_new"], stg.dev["slot_mapping"], stg.dev["q"], dev.k_cache,
                      dev.v_cache, stg.dev["block_tables"], stg.dev["context_lens"], case.scale, dev.out)
    stg.download(dev.out)
    dec.append_decode(ref.k_new, ref.v_new, ref.slot_mapping, ref.q, ref.k_cache, ref.v_cache, ref.block_tables,
                      ref.context_lens, case.scale, ref.out)
    torch.cuda.synchronize()
    assert dec.device_error() == 0
    assert torch.equal(stg.out, ref.out.cpu())
    assert torch.equal(dev.k_cache, ref.k_cache) and torch.equal(dev.v_cache, ref.v_cache)
    H.assert_close(stg.out.float().numpy().astype(np.float64), oracle_out(orc, case), case.dtype, "staged")
