"""The seeded input generator (CPU only): known-answer values of its random
number generator and the structure of the five decode workloads."""
import numpy as np
import pytest

import synth
from synth.workloads import bf16_bits_to_f32, f32_to_bf16_bits, normals, philox4x32_10


def test_philox_known_answers():
    # Known-answer vectors of Philox4x32-10 (Salmon et al., SC 2011).
    assert list(philox4x32_10([0, 0, 0, 0], [0, 0])) == [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]
    ff = 0xFFFFFFFF
    assert list(philox4x32_10([ff] * 4, [ff] * 2)) == [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]


def test_normals_moments_and_determinism():
    a = normals(123, 0, (1 << 20,), "f32")
    b = normals(123, 0, (1 << 20,), "f32")
    c = normals(123, 1, (1 << 20,), "f32")
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    assert abs(a.mean()) < 5e-3 and abs(a.std() - 1.0) < 5e-3
    assert abs((np.abs(a) < 1.0).mean() - 0.6827) < 3e-3


def test_bf16_rounding_nearest_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.5, 1.0 + 2**-9, 1.0 + 2**-8 + 2**-20], np.float32)
    back = bf16_bits_to_f32(f32_to_bf16_bits(x))
    # bf16 spacing at 1.0 is 2^-7: exact halves go to the even mantissa
    expect = np.array([1.0, 1.0, 1.0 + 2**-6, -2.5, 1.0, 1.0 + 2**-7], np.float32)
    assert np.array_equal(back, expect)
    assert normals(5, 0, (64,), "bf16").dtype == np.uint16


@pytest.mark.parametrize("cid", [1, 2, 3, 4, 5])
def test_config_structure(cid):
    c = synth.make_config(cid, values=False)
    lo, hi = {1: (17, 33), 2: (128, 2048), 3: (512, 4096), 4: (32768, 131072), 5: (16, 16384)}[cid]
    assert c.context_lens.min() >= lo and c.context_lens.max() <= hi
    assert c.B == {1: 2, 2: 32, 3: 128, 4: 8, 5: 256}[cid]
    bs = c.block_size
    used = []
    for b in range(c.B):
        L = int(c.context_lens[b])
        n = -(-L // bs)
        row = c.block_tables[b]
        assert np.all(row[:n] >= 0) and np.all(row[:n] < c.num_blocks)
        assert np.all(row[n:] == -1)
        pos = L - 1
        assert c.slot_mapping[b] == row[pos // bs] * bs + pos % bs
        used.extend(int(x) for x in row[:n])
    if cid == 5:
        # first full blocks are shared inside each group of 8; append slots stay private
        for gk in range(0, c.B, 8):
            for b in range(gk, gk + 8):
                ns = min(4, (int(c.context_lens[b]) - 1) // bs)
                ref = [b2 for b2 in range(gk, gk + 8) if min(4, (int(c.context_lens[b2]) - 1) // bs) >= ns]
                for b2 in ref:
                    assert np.array_equal(c.block_tables[b, :ns], c.block_tables[b2, :ns])
        slots_blocks = set(int(s) // bs for s in c.slot_mapping)
        assert len(slots_blocks) == c.B
        assert c.unique_blocks() < c.blocks_used()
    else:
        assert len(set(used)) == len(used)        # no block is shared
    if cid == 3:
        assert c.num_blocks == int(np.ceil(1.5 * c.blocks_used()))
    if cid == 1:
        assert c.num_blocks == 8 and c.dtype == "f32"
    if cid == 4:
        assert c.partition_tokens == 512 and c.Hkv == 1 and c.block_size == 256


def test_config_is_deterministic():
    a = synth.make_config(1)
    b = synth.make_config(1)
    for f in ("q", "k_new", "v_new", "k_cache", "v_cache", "block_tables", "slot_mapping", "context_lens"):
        assert np.array_equal(getattr(a, f), getattr(b, f))


@pytest.mark.parametrize("pid", [1, 2])
def test_prefill_config_structure(pid):
    pc = synth.make_prefill_config(pid, values=False)
    qs = pc.query_start.astype(np.int64)
    n = np.diff(qs)
    assert qs[0] == 0 and qs[-1] == pc.T and np.all(n >= 1) and np.all(n <= pc.context_lens)
    pos = pc.positions()
    for b in range(pc.B):
        L = int(pc.context_lens[b])
        nblk = -(-L // pc.block_size)
        assert np.all((pc.block_tables[b, :nblk] >= 0) & (pc.block_tables[b, :nblk] < pc.num_blocks))
        for i in range(qs[b], qs[b + 1]):
            assert pos[i] == L - n[b] + (i - qs[b])
            p_ = int(pos[i])
            assert pc.slot_mapping[i] == pc.block_tables[b, p_ // pc.block_size] * pc.block_size + p_ % pc.block_size
    assert len(set(pc.slot_mapping.tolist())) == pc.T          # distinct slots
    again = synth.make_prefill_config(pid, values=False)
    assert np.array_equal(again.context_lens, pc.context_lens) and np.array_equal(again.slot_mapping, pc.slot_mapping)


def test_prefill_algorithmic_counts_by_brute_force():
    """The prefill metric's flops and bytes, recounted pair by pair on a small case."""
    pc = synth.build_prefill_case("count", dtype="bf16", Hq=8, Hkv=2, D=64, block_size=16,
                                  context_lens=[40, 7, 100], new_tokens=[40, 3, 17], seed=5, values=False,
                                  pool="factor", pool_factor=1.5)
    pairs = 0
    for b in range(pc.B):
        L, n = int(pc.context_lens[b]), int(pc.query_start[b + 1] - pc.query_start[b])
        for j in range(n):
            pos = L - n + j
            pairs += sum(1 for t in range(L) if t <= pos)
    alg = synth.prefill_algorithmic(pc)
    assert alg["flops"] == 4 * pairs * pc.Hq * pc.D
    assert alg["bytes"] == int(sum(pc.context_lens)) * pc.Hkv * pc.D * 2 * 2 + 2 * pc.T * pc.Hq * pc.D * 2


@pytest.mark.parametrize("cid", [1, 2, 3, 4, 5])
def test_decode_algorithmic_bytes_by_definition(cid):
    """The decode metric's bytes recounted from the lengths: K and V of every
    position each request reads, q in and out, one table entry per block used
    and one length per request."""
    case = synth.make_config(cid, values=False)
    e = {"f32": 4, "bf16": 2, "f16": 2}[case.dtype]
    L = [int(x) for x in case.context_lens]
    kv = sum(l * case.Hkv * case.D * e * 2 for l in L)
    qo = 2 * case.B * case.Hq * case.D * e
    tables = 4 * sum(-(-l // case.block_size) for l in L) + 4 * case.B
    a = synth.algorithmic_bytes(case)
    assert a["kv"] == kv and a["q_out"] == qo and a["tables"] == tables
    assert a["decode_total"] == kv + qo + tables
