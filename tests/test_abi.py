"""The C ABI without a GPU: the library loads, exports every declared symbol,
plans the five workloads, and rejects bad arguments with a status (never a
crash).  No call here launches a kernel."""
import ctypes
import os
import re

import pytest

import __graft_entry__

__graft_entry__.build()
import paged_kv_cache_472_b200 as pa  # noqa: E402
import synth  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names.update(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert len(names) >= 10, names
    for n in names:
        assert hasattr(pa.lib, n), n


def test_status_strings_and_version():
    assert pa.pa_status_str(0) == "PA_OK"
    assert pa.pa_status_str(4) == "PA_ERR_WORKSPACE"
    assert pa.pa_version() >= 100


def shape_of(case):
    return pa.Shape(case.B, case.Hq, case.Hkv, case.D, case.block_size, case.num_blocks,
                    case.max_blocks_per_seq, pa.DTYPE_F32 if case.dtype == "f32" else pa.DTYPE_BF16)


@pytest.mark.parametrize("cid", [1, 2, 3, 4, 5])
def test_plan_workloads(cid):
    c = synth.make_config(cid, values=False)
    s = shape_of(c)
    plan = pa.pa_plan(s, int(c.max_blocks_per_seq * c.block_size), c.partition_tokens, 148)
    G = c.Hq // c.Hkv
    assert plan.num_ctas == 148
    assert plan.smem_bytes <= 232448 - 256
    assert plan.stages >= 2
    assert plan.head_group * plan.heads_per_unit >= 1
    units = plan.head_group * G // plan.heads_per_unit
    if plan.heads_per_unit >= 16:      # tcgen05 engine: one KV head, all its query heads in one tile
        assert (plan.head_group, plan.heads_per_unit, plan.tile_tokens) == (1, G, 128)
    else:
        assert units == 8 * plan.units_per_warp or units * plan.warps_per_unit == 8
    assert plan.tile_tokens >= 16 and plan.tile_tokens & (plan.tile_tokens - 1) == 0
    assert pa.pa_decode_workspace_size(plan) == plan.workspace_bytes
    if c.partition_tokens:
        assert plan.mode == pa.SPLIT_FIXED and plan.partition_tokens % plan.tile_tokens == 0
    else:
        # static piece (vr v, slice r) -> slot v + r; dynamic piece (vr v, grain j) -> NV + C + v + j,
        # with at most 8*C*share/256 + 1 grains
        NV = c.B * (c.Hkv // plan.head_group)
        assert plan.mode == pa.SPLIT_BALANCED and plan.dynamic_share == 0
        assert plan.max_slots == 2 * NV + 148 + 8 * 148 * 64 // 256 + 1
    assert plan.split_merge == (1 if cid in (1, 4) else 0)   # few (request, KV head group) pairs per CTA
    expect = {1: (2, 1, 2), 2: (8, 2, 1), 3: (8, 4, 1), 4: (1, 32, 1), 5: (8, 4, 1)}[cid]
    assert (plan.head_group, plan.heads_per_unit, plan.warps_per_unit) == expect


@pytest.mark.parametrize("Hq,Hkv,D,upw,hc,hg,ts", [
    (32, 32, 128, 1, 1, 8, 1), (16, 16, 64, 2, 1, 16, 1), (64, 16, 64, 2, 4, 16, 1), (32, 16, 64, 2, 2, 16, 1),
    (64, 16, 128, 1, 4, 8, 1), (4, 1, 128, 1, 4, 1, 8), (8, 1, 128, 1, 8, 1, 8), (64, 1, 128, 1, 64, 1, 1),
    (2, 2, 64, 1, 1, 2, 4), (1, 1, 64, 1, 1, 1, 8), (32, 1, 128, 1, 32, 1, 1), (32, 2, 128, 1, 16, 1, 1),
    (32, 1, 64, 1, 8, 1, 2), (64, 1, 64, 1, 8, 1, 1)])
def test_plan_head_mappings(Hq, Hkv, D, upw, hc, hg, ts):
    """bf16 shapes use the tensor-core engines: with D = 128 and 16, 32 or 64 query heads per KV head,
    the tcgen05 engine (one KV head per work item, all its query heads in one tile); otherwise warp-level
    tiles, a unit being one KV head with up to 8 query heads."""
    s = pa.Shape(3, Hq, Hkv, D, 16, 64, 8, pa.DTYPE_BF16)
    plan = pa.pa_plan(s, 128, 0, 148)
    assert (plan.units_per_warp, plan.heads_per_unit, plan.head_group, plan.warps_per_unit) == (upw, hc, hg, ts)


@pytest.mark.parametrize("Hq,Hkv,D,upw,hc,hg,ts", [
    (4, 2, 64, 1, 1, 2, 2), (16, 4, 128, 1, 2, 4, 1), (8, 2, 64, 1, 1, 2, 1), (1, 1, 64, 1, 1, 1, 8),
    (32, 32, 64, 1, 1, 8, 1)])
def test_plan_head_mappings_fp32(Hq, Hkv, D, upw, hc, hg, ts):
    """fp32 shapes use the CUDA-core engine."""
    s = pa.Shape(3, Hq, Hkv, D, 16, 64, 8, pa.DTYPE_F32)
    plan = pa.pa_plan(s, 128, 0, 148)
    assert (plan.units_per_warp, plan.heads_per_unit, plan.head_group, plan.warps_per_unit) == (upw, hc, hg, ts)


@pytest.mark.parametrize("mut,status", [
    (dict(D=96), pa.PA_ERR_UNSUPPORTED), (dict(block_size=8), pa.PA_ERR_UNSUPPORTED),
    (dict(block_size=48), pa.PA_ERR_UNSUPPORTED), (dict(Hq=12, Hkv=4), pa.PA_ERR_UNSUPPORTED),
    (dict(Hq=10, Hkv=4), pa.PA_ERR_INVALID_ARG), (dict(dtype=7), pa.PA_ERR_INVALID_ARG),
    (dict(B=-1), pa.PA_ERR_INVALID_ARG), (dict(num_blocks=0), pa.PA_ERR_INVALID_ARG),
])
def test_plan_rejects(mut, status):
    base = dict(B=2, Hq=8, Hkv=2, D=128, block_size=16, num_blocks=8, max_blocks_per_seq=4, dtype=pa.DTYPE_BF16)
    base.update(mut)
    s = pa.Shape(**base)
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.pa_plan(s, 32, 0, 148)
    assert ei.value.status == status


def test_plan_rejects_bad_partition_and_context():
    s = pa.Shape(2, 8, 2, 128, 16, 8, 4, pa.DTYPE_BF16)
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.pa_plan(s, 32, 10, 148)
    assert ei.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.pa_plan(s, 65, 0, 148)          # > max_blocks_per_seq * block_size
    assert ei.value.status == pa.PA_ERR_INVALID_ARG


def test_tcgen05_engine_needs_whole_tiles_per_partition():
    """Fixed partitions that are not a multiple of the 128-token tile keep the warp-level engine."""
    s = pa.Shape(2, 32, 1, 128, 256, 64, 16, pa.DTYPE_BF16)
    assert pa.pa_plan(s, 4096, 512, 148).heads_per_unit == 32
    assert pa.pa_plan(s, 4096, 0, 148).heads_per_unit == 32
    p64 = pa.pa_plan(s, 4096, 64, 148)
    assert (p64.heads_per_unit, p64.warps_per_unit) == (8, 2)
    for G, stages in ((16, 3), (32, 3), (64, 2)):
        p = pa.pa_plan(pa.Shape(2, G, 1, 128, 16, 64, 16, pa.DTYPE_F16), 256, 0, 148)
        assert (p.heads_per_unit, p.tile_tokens, p.stages) == (G, 128, stages)
        assert p.smem_bytes <= 232448 - 10 * 1024


def test_fixed_plan_workspace_formula():
    s = pa.Shape(8, 32, 1, 128, 256, 4096, 512, pa.DTYPE_BF16)
    plan = pa.pa_plan(s, 131072, 512, 148)
    assert plan.max_slots == 8 + 148          # one partial per (request, slice)
    slot_floats = 32 * 128 + 64
    assert plan.split_merge == 1                # 148 CTAs over 8 requests: a merge grid combines the pieces
    assert plan.workspace_bytes == 256 + 256 + 256 + plan.max_slots * slot_floats * 4   # + the merge records


FAKE = 1 << 20  # aligned, never dereferenced: every call below fails validation first


def _decode(s, plan, **kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, tables=FAKE, lens=FAKE, scale=0.1, out=FAKE, ws=FAKE,
                ws_bytes=plan.workspace_bytes if plan else 0)
    args.update(kw)
    return pa.lib.pa_decode(args["q"], args["k"], args["v"], args["tables"], args["lens"], args["scale"], args["out"],
                            ctypes.byref(s), ctypes.byref(plan) if plan else None, args["ws"], args["ws_bytes"], None)


def test_decode_validation_paths():
    s = pa.Shape(2, 8, 2, 128, 16, 8, 4, pa.DTYPE_BF16)
    plan = pa.pa_plan(s, 64, 0, 148)
    assert _decode(s, None) == pa.PA_ERR_INVALID_ARG
    assert _decode(s, plan, ws_bytes=plan.workspace_bytes - 1) == pa.PA_ERR_WORKSPACE
    assert _decode(s, plan, ws=0) == pa.PA_ERR_WORKSPACE
    assert _decode(s, plan, ws=FAKE + 16) == pa.PA_ERR_INVALID_ARG        # not 256-aligned
    assert _decode(s, plan, q=FAKE + 2) == pa.PA_ERR_INVALID_ARG          # not 16-aligned
    plan.flags = 0x100                                                    # unknown flag bit
    assert _decode(s, plan) == pa.PA_ERR_INVALID_ARG
    plan.flags = pa.PLAN_NO_SPECULATION | pa.PLAN_TEST_MISGUESS
    assert _decode(s, plan, ws=0) == pa.PA_ERR_WORKSPACE                  # known bits pass on to later checks
    plan.flags = 0
    assert _decode(s, plan, out=0) == pa.PA_ERR_INVALID_ARG
    assert _decode(s, plan, scale=float("nan")) == pa.PA_ERR_INVALID_ARG
    s2 = pa.Shape(2, 8, 2, 128, 16, 9, 4, pa.DTYPE_BF16)                 # plan made for another shape
    assert _decode(s2, plan) == pa.PA_ERR_INVALID_ARG
    s0 = pa.Shape(0, 8, 2, 128, 16, 8, 4, pa.DTYPE_BF16)
    plan0 = pa.pa_plan(s0, 64, 0, 148)
    assert _decode(s0, plan0) == pa.PA_OK                                 # empty batch: nothing to launch
    assert "plan" in pa.pa_last_error_message() or pa.pa_last_error_message() == ""


def test_append_validation_paths():
    s = pa.Shape(2, 8, 2, 128, 16, 8, 4, pa.DTYPE_BF16)
    f = pa.lib.pa_kv_append
    assert f(FAKE, FAKE, FAKE, FAKE, 0, ctypes.byref(s), None, None) == pa.PA_ERR_INVALID_ARG
    assert f(FAKE + 4, FAKE, FAKE, FAKE, FAKE, ctypes.byref(s), None, None) == pa.PA_ERR_INVALID_ARG
    s0 = pa.Shape(0, 8, 2, 128, 16, 8, 4, pa.DTYPE_BF16)
    assert f(0, 0, 0, 0, 0, ctypes.byref(s0), None, None) == pa.PA_OK
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None) == pa.PA_ERR_INVALID_ARG


@pytest.mark.parametrize("share,mode_fixed", [(-1, False), (65, False), (16, True)])
def test_decode_rejects_bad_dynamic_share(share, mode_fixed):
    """The plan's dynamic share is checked before anything reaches the GPU."""
    s = pa.Shape(2, 8, 2, 128, 16, 8, 4, pa.DTYPE_BF16)
    plan = pa.pa_plan(s, 64, 16 if mode_fixed else 0, 148)
    plan.dynamic_share = share
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.pa_decode(0, 0, 0, 0, 0, 0.1, 0, s, plan, 0, 0, stream=0)
    assert ei.value.status == pa.PA_ERR_INVALID_ARG


def test_prefill_plan_shapes_and_rejections():
    s = pa.Shape(8, 32, 8, 128, 16, 4096, 256, pa.DTYPE_BF16)
    plan = pa.pa_prefill_plan(s, 512)
    assert plan.q_tile * 4 == 128 and plan.num_qtiles == 512 // (2 * plan.q_tile) and plan.stages >= 2
    assert plan.smem_bytes <= 232448
    for bad, status in ((pa.Shape(2, 8, 2, 128, 16, 64, 8, pa.DTYPE_F32), pa.PA_ERR_UNSUPPORTED),
                        (pa.Shape(2, 8, 2, 96, 16, 64, 8, pa.DTYPE_BF16), pa.PA_ERR_UNSUPPORTED),
                        (pa.Shape(2, 8, 2, 128, 8, 64, 8, pa.DTYPE_BF16), pa.PA_ERR_UNSUPPORTED),
                        (pa.Shape(2, 6, 2, 128, 16, 64, 8, pa.DTYPE_BF16), pa.PA_ERR_UNSUPPORTED)):
        with pytest.raises(pa.PagedAttnError) as ei:
            pa.pa_prefill_plan(bad, 16)
        assert ei.value.status == status
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.pa_prefill_plan(s, 256 * 16 + 1)            # more new tokens than a table row holds
    assert ei.value.status == pa.PA_ERR_INVALID_ARG


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", [pa.DTYPE_BF16, pa.DTYPE_F16])
def test_prefill_plan_budget_over_supported_shapes(D, dtype):
    """Every supported shape gets a plan that fits the 227 KB shared-memory limit
    with at least one K and one V slot, and tiles of 128 rows."""
    for G in (1, 2, 4, 8, 16, 32, 64, 128):
        for bs in (16, 32, 64, 128, 256):
            s = pa.Shape(3, G * 2, 2, D, bs, 64, 16, dtype)
            plan = pa.pa_prefill_plan(s, 100)
            assert plan.q_tile * G == 128 and plan.kv_tile == 128
            assert 2 <= 2 * plan.stages and plan.smem_bytes + 3072 <= 232448
            assert plan.num_qtiles == -(-100 // (2 * plan.q_tile))   # two query tiles per CTA


@pytest.mark.parametrize("field,value", [("head_group", 0), ("head_group", 3), ("stages", 9), ("tile_tokens", 48),
                                         ("smem_bytes", 1024), ("workspace_bytes", 512), ("max_slots", 1),
                                         ("num_ctas", 0), ("units_per_warp", 3), ("mode", 7),
                                         ("max_context_len", 10**6)])
def test_decode_rejects_a_tampered_plan(field, value):
    """Every plan field the launch derives anything from is checked against the
    planner's own output before anything is queued (host only, no GPU)."""
    s = pa.Shape(4, 16, 8, 128, 16, 64, 16, pa.DTYPE_BF16)
    plan = pa.pa_plan(s, 256, 0, 148)
    setattr(plan, field, value)
    assert _decode(s, plan, ws_bytes=1 << 30) == pa.PA_ERR_INVALID_ARG
    assert "plan" in pa.pa_last_error_message()


def test_no_alloc_rejects_a_stale_plan_before_touching_its_array():
    """A plan made for one request passed with a 4096-request shape: rejected on
    the host, before the built-in array is looked up or cleared (this runs
    without a GPU, so any device call would fail with PA_ERR_CUDA instead)."""
    s1 = pa.Shape(1, 32, 8, 128, 16, 70000, 64, pa.DTYPE_BF16)
    plan = pa.pa_plan(s1, 1024, 0, 148)
    big = pa.Shape(4096, 32, 8, 128, 16, 70000, 64, pa.DTYPE_BF16)
    st = pa.lib.pa_decode_no_alloc(FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.1), FAKE, ctypes.byref(big),
                                   ctypes.byref(plan), None)
    assert st == pa.PA_ERR_INVALID_ARG
    plan.head_group = 0                                    # tampered: would divide by zero
    st = pa.lib.pa_decode_no_alloc(FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.1), FAKE, ctypes.byref(s1),
                                   ctypes.byref(plan), None)
    assert st == pa.PA_ERR_INVALID_ARG


def test_stall_flag_is_a_known_flag():
    s = pa.Shape(2, 8, 2, 128, 16, 8, 4, pa.DTYPE_BF16)
    plan = pa.pa_plan(s, 64, 0, 148)
    plan.flags = pa.PLAN_TEST_STALL
    assert _decode(s, plan, ws=0) == pa.PA_ERR_WORKSPACE       # passes the flag check
    plan.flags = 0x8
    assert _decode(s, plan) == pa.PA_ERR_INVALID_ARG
