"""The float64 oracle against its pins (CPU only)."""
import numpy as np
import pytest

import synth
from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_rejects_table_entry_outside_pool(orc):
    case = synth.make_config(1)
    bad = case.block_tables.copy()
    bad[1, 2] = case.num_blocks          # one past the pool
    with pytest.raises(ValueError):
        orc.decode(case, case.k_cache, case.v_cache, block_tables=bad)


def test_rejects_context_longer_than_table(orc):
    case = synth.make_config(1)
    lens = case.context_lens.copy()
    lens[0] = case.max_blocks_per_seq * case.block_size + 1
    with pytest.raises(ValueError):
        orc.decode(case, case.k_cache, case.v_cache, context_lens=lens)


def test_rejects_append_slot_outside_pool(orc):
    case = synth.make_config(1)
    case.slot_mapping = case.slot_mapping.copy()
    case.slot_mapping[1] = case.num_blocks * case.block_size
    with pytest.raises(ValueError):
        orc.kv_append(case)


def test_zero_length_context_gives_zero(orc):
    case = synth.build_case("len0", dtype="f32", Hq=2, Hkv=1, D=4, block_size=4, context_lens=[3, 1],
                            seed=5)
    kc, vc = orc.kv_append(case)
    lens = case.context_lens.copy()
    lens[1] = 0
    out = orc.decode(case, kc, vc, context_lens=lens)
    assert np.all(out[1] == 0.0)


def test_pairs_match_full_decode(orc):
    case = synth.make_config(1)
    kc, vc = orc.kv_append(case)
    full = orc.decode(case, kc, vc)
    pairs = [(1, 3), (0, 0), (1, 0)]
    sub = orc.decode_pairs(case, pairs, kc, vc)
    for i, (b, h) in enumerate(pairs):
        assert np.array_equal(sub[i], full[b, h])


def test_thread_count_does_not_change_result(orc):
    case = synth.make_config(1)
    kc, vc = orc.kv_append(case)
    assert np.array_equal(orc.decode(case, kc, vc, nthreads=1), orc.decode(case, kc, vc, nthreads=4))


def test_fp16_values_widen_exactly(orc):
    """Every finite fp16 bit pattern reaches the oracle's arithmetic exactly:
    with one token, out = V, compared with numpy's float16 -> float64."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = bits[np.isfinite(bits.view(np.float16))]
    D = 256
    n = -(-finite.size // D) * D
    vals = np.zeros(n, np.uint16)
    vals[:finite.size] = finite
    rows = n // D
    case = synth.build_case("f16bits", dtype="f16", Hq=1, Hkv=1, D=D, block_size=16,
                            context_lens=[1] * rows, seed=4)
    case.v_new = vals.reshape(rows, 1, D)
    out = orc.decode(case)
    want = vals.view(np.float16).astype(np.float64).reshape(rows, 1, D)
    assert np.array_equal(out, want)


def test_prefill_rows_match_full_prefill(orc):
    pc = synth.make_prefill_config(2, batch=3, chunk=40)
    full = orc.prefill(pc)
    rows = [0, 5, pc.T - 1, int(pc.query_start[1])]
    assert np.array_equal(orc.prefill_rows(pc, rows), full[rows])
