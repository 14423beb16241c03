"""Pins that tie the float64 oracle to what the pages and the mathematics fix.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with something that does not come from the oracle itself:
  * hand-derived closed-form cases in tests/golden (rules the pages state);
  * brute force in plain Python loops on tiny inputs;
  * an independent numpy float64 dense attention over a gathered cache;
  * invariants the pages state or imply: paged == contiguous storage,
    GQA/MQA == MHA with repeated KV heads, physical block ids can be permuted,
    one token returns V, identical keys return the mean of V,
    partition + log-sum-exp merge == unsplit;
  * for chunked prefill: brute force, one new token == decode, a fresh
    request's first token returns its own V, causality (a later token's K/V
    never reaches an earlier token).
The same pins run against deliberately broken copies of the oracle
(tests/test_oracle_mutants.py), so each plausible slip fails at least one.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import synth
from synth import DTYPE_BF16, DTYPE_F32, PagedDecodeCase, build_case

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def case_from_fixture(fx) -> PagedDecodeCase:
    Hq, Hkv, D, bs, nb = fx["Hq"], fx["Hkv"], fx["D"], fx["block_size"], fx["num_blocks"]
    k = np.full((nb, bs, Hkv, D), fx["fill"], dtype=np.float32)
    v = np.full((nb, bs, Hkv, D), fx["fill"], dtype=np.float32)
    for key, rows in fx["k_rows"].items():
        blk, row = map(int, key.split(","))
        k[blk, row] = np.asarray(rows, np.float32)
    for key, rows in fx["v_rows"].items():
        blk, row = map(int, key.split(","))
        v[blk, row] = np.asarray(rows, np.float32)
    tables = np.asarray(fx["block_tables"], np.int32)
    lens = np.asarray(fx["context_lens"], np.int32)
    B = lens.shape[0]
    z = np.zeros((B, Hkv, D), np.float32)
    return PagedDecodeCase(name=fx["name"], dtype=DTYPE_F32, B=B, Hq=Hq, Hkv=Hkv, D=D, block_size=bs,
                           num_blocks=nb, max_blocks_per_seq=tables.shape[1], context_lens=lens,
                           block_tables=tables, slot_mapping=np.full(B, -1, np.int32),
                           q=np.asarray(fx["q"], np.float32), k_new=z, v_new=z.copy(), k_cache=k,
                           v_cache=v, scale=float(fx["scale"]))


def _f64(case, a):
    return case.as_float32(a).astype(np.float64)


def tiny_cases():
    """Small seeded cases covering fp32/bf16, MHA/GQA/MQA, D in {8, 64},
    block sizes 1..16, lengths 1, bs, bs +- 1 and several blocks."""
    specs = [
        dict(dtype=DTYPE_F32, Hq=4, Hkv=2, D=8, block_size=4, context_lens=[5, 9, 1, 4], seed=11),
        dict(dtype=DTYPE_BF16, Hq=4, Hkv=1, D=8, block_size=2, context_lens=[3, 7], seed=12),
        dict(dtype=DTYPE_BF16, Hq=3, Hkv=3, D=4, block_size=1, context_lens=[2, 1, 6], seed=13),
        dict(dtype=DTYPE_F32, Hq=8, Hkv=2, D=16, block_size=16, context_lens=[15, 16, 17, 33], seed=14,
             pool="factor", pool_factor=1.5),
    ]
    return [build_case(f"tiny{i}", **s) for i, s in enumerate(specs)]


def brute_force(case, k_cache, v_cache):
    """Plain-Python softmax attention, one (request, head) at a time."""
    q = _f64(case, case.q)
    K = _f64(case, k_cache)
    V = _f64(case, v_cache)
    G = case.Hq // case.Hkv
    out = np.zeros((case.B, case.Hq, case.D))
    for b in range(case.B):
        L = int(case.context_lens[b])
        for h in range(case.Hq):
            g = h // G
            rows = []
            for t in range(L):
                phys = int(case.block_tables[b][t // case.block_size])
                rows.append((phys, t % case.block_size))
            s = []
            for (p, o) in rows:
                acc = 0.0
                for d in range(case.D):
                    acc += float(q[b, h, d]) * float(K[p, o, g, d])
                s.append(case.scale * acc)
            m = max(s)
            w = [math.exp(x - m) for x in s]
            tot = sum(w)
            for d in range(case.D):
                out[b, h, d] = sum(w[i] * float(V[p, o, g, d]) for i, (p, o) in enumerate(rows)) / tot
    return out


def dense_numpy(case, k_cache, v_cache):
    """Gather each request's pages into a dense [L, Hkv, D] array, then run a
    textbook dense softmax attention with numpy in float64."""
    q = _f64(case, case.q)
    K = _f64(case, k_cache)
    V = _f64(case, v_cache)
    G = case.Hq // case.Hkv
    out = np.zeros((case.B, case.Hq, case.D))
    for b in range(case.B):
        L = int(case.context_lens[b])
        idx = [(int(case.block_tables[b][t // case.block_size]), t % case.block_size) for t in range(L)]
        Kd = np.stack([K[p, o] for p, o in idx])          # [L, Hkv, D]
        Vd = np.stack([V[p, o] for p, o in idx])
        Kr = np.repeat(Kd, G, axis=1)                      # [L, Hq, D]
        Vr = np.repeat(Vd, G, axis=1)
        s = np.einsum("hd,lhd->hl", q[b], Kr) * case.scale
        w = np.exp(s - s.max(axis=1, keepdims=True))
        out[b] = np.einsum("hl,lhd->hd", w, Vr) / w.sum(axis=1)[:, None]
    return out


def _appended(orc, case):
    return orc.kv_append(case)


# ----------------------------------------------------------------------------
def pin_golden_decode(orc):
    for fx in _load("decode_closed_form.json")["cases"]:
        case = case_from_fixture(fx)
        out = orc.decode(case, case.k_cache, case.v_cache)
        np.testing.assert_allclose(out, np.asarray(fx["expected"]), rtol=1e-14, atol=1e-15,
                                   err_msg=fx["name"])


def pin_golden_append(orc):
    for fx in _load("append_closed_form.json")["cases"]:
        Hkv, D, bs, nb = fx["Hkv"], fx["D"], fx["block_size"], fx["num_blocks"]
        slots = np.asarray(fx["slot_mapping"], np.int32)
        B = slots.shape[0]
        case = PagedDecodeCase(name=fx["name"], dtype=DTYPE_F32, B=B, Hq=Hkv, Hkv=Hkv, D=D, block_size=bs,
                               num_blocks=nb, max_blocks_per_seq=1, context_lens=np.zeros(B, np.int32),
                               block_tables=np.zeros((B, 1), np.int32), slot_mapping=slots,
                               q=np.zeros((B, Hkv, D), np.float32),
                               k_new=np.asarray(fx["k_new"], np.float32), v_new=np.asarray(fx["v_new"], np.float32),
                               k_cache=np.zeros((nb, bs, Hkv, D), np.float32),
                               v_cache=np.zeros((nb, bs, Hkv, D), np.float32), scale=1.0)
        kc, vc = orc.kv_append(case)
        ek = np.zeros_like(kc)
        ev = np.zeros_like(vc)
        for key, rows in fx["expected_rows"].items():
            blk, row = map(int, key.split(","))
            ek[blk, row] = np.asarray(rows["k"], np.float32)
            ev[blk, row] = np.asarray(rows["v"], np.float32)
        assert np.array_equal(kc, ek), fx["name"]
        assert np.array_equal(vc, ev), fx["name"]


def pin_brute_force(orc):
    for case in tiny_cases():
        kc, vc = _appended(orc, case)
        out = orc.decode(case, kc, vc)
        ref = brute_force(case, kc, vc)
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13, err_msg=case.name)


def pin_dense_numpy(orc):
    cases = tiny_cases() + [synth.make_config(1)]
    for case in cases:
        kc, vc = _appended(orc, case)
        out = orc.decode(case, kc, vc)
        ref = dense_numpy(case, kc, vc)
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13, err_msg=case.name)


def _contiguous_copy(case, kc, vc):
    """Same logical cache with every request's blocks stored in order."""
    nblk = [-(-int(L) // case.block_size) for L in case.context_lens]
    total = sum(nblk)
    k2 = np.zeros((max(total, 1),) + kc.shape[1:], kc.dtype)
    v2 = np.zeros_like(k2)
    t2 = np.full_like(case.block_tables, -1)
    nxt = 0
    for b in range(case.B):
        for j in range(nblk[b]):
            p = int(case.block_tables[b][j])
            k2[nxt], v2[nxt] = kc[p], vc[p]
            t2[b][j] = nxt
            nxt += 1
    return k2, v2, t2


def pin_paged_equals_contiguous(orc):
    for case in tiny_cases() + [synth.make_config(1)]:
        kc, vc = _appended(orc, case)
        out = orc.decode(case, kc, vc)
        k2, v2, t2 = _contiguous_copy(case, kc, vc)
        out2 = orc.decode(case, k2, v2, block_tables=t2)
        assert np.array_equal(out, out2), case.name


def pin_gqa_equals_repeated_mha(orc):
    for case in tiny_cases() + [synth.make_config(1)]:
        G = case.Hq // case.Hkv
        if G == 1:
            continue
        kc, vc = _appended(orc, case)
        out = orc.decode(case, kc, vc)
        mha = PagedDecodeCase(**{**case.__dict__, "Hkv": case.Hq})
        out2 = orc.decode(mha, np.repeat(kc, G, axis=2), np.repeat(vc, G, axis=2))
        assert np.array_equal(out, out2), case.name


def pin_block_permutation(orc):
    rng = np.random.default_rng(7)
    for case in tiny_cases() + [synth.make_config(1)]:
        kc, vc = _appended(orc, case)
        out = orc.decode(case, kc, vc)
        perm = rng.permutation(kc.shape[0])
        k2 = np.empty_like(kc)
        v2 = np.empty_like(vc)
        k2[perm] = kc
        v2[perm] = vc
        t2 = np.where(case.block_tables >= 0, perm[np.maximum(case.block_tables, 0)], -1).astype(np.int32)
        out2 = orc.decode(case, k2, v2, block_tables=t2)
        assert np.array_equal(out, out2), case.name


def pin_single_token_returns_v(orc):
    for dtype in (DTYPE_F32, DTYPE_BF16):
        case = build_case("len1", dtype=dtype, Hq=6, Hkv=3, D=8, block_size=4, context_lens=[1, 1, 1],
                          seed=21)
        kc, vc = _appended(orc, case)
        out = orc.decode(case, kc, vc)
        vnew = _f64(case, case.v_new)
        G = case.Hq // case.Hkv
        for b in range(case.B):
            for h in range(case.Hq):
                assert np.array_equal(out[b, h], vnew[b, h // G]), (dtype, b, h)


def pin_identical_keys_mean_v(orc):
    for dtype in (DTYPE_F32, DTYPE_BF16):
        case = build_case("samekey", dtype=dtype, Hq=4, Hkv=2, D=8, block_size=4, context_lens=[7, 12],
                          seed=22)
        kc, vc = _appended(orc, case)
        kc = np.broadcast_to(kc[0, 0, 0], kc.shape).copy()   # every key row equal
        out = orc.decode(case, kc, vc)
        V = _f64(case, vc)
        G = case.Hq // case.Hkv
        for b in range(case.B):
            L = int(case.context_lens[b])
            for h in range(case.Hq):
                rows = [V[int(case.block_tables[b][t // case.block_size]), t % case.block_size, h // G]
                        for t in range(L)]
                np.testing.assert_allclose(out[b, h], np.mean(rows, axis=0), rtol=1e-13, atol=1e-14)


def pin_partitioned_equals_unsplit(orc):
    for case in tiny_cases() + [synth.make_config(1)]:
        kc, vc = _appended(orc, case)
        out = orc.decode(case, kc, vc)
        for part in (1, 2, 3, 16, 17, 10000):
            outp = orc.decode_partitioned(case, part, kc, vc)
            np.testing.assert_allclose(outp, out, rtol=1e-12, atol=1e-13, err_msg=f"{case.name} part={part}")


def pin_append_matches_index_assignment(orc):
    for case in tiny_cases() + [synth.make_config(1)]:
        case.slot_mapping = case.slot_mapping.copy()
        case.slot_mapping[0] = -1                      # one request does not append
        kc, vc = orc.kv_append(case)
        ek = case.k_cache.copy().reshape(-1, case.Hkv, case.D)
        ev = case.v_cache.copy().reshape(-1, case.Hkv, case.D)
        for i, s in enumerate(case.slot_mapping):
            if s >= 0:
                ek[s] = case.k_new[i]
                ev[s] = case.v_new[i]
        assert np.array_equal(kc.reshape(ek.shape).view(np.uint8), ek.view(np.uint8)), case.name
        assert np.array_equal(vc.reshape(ev.shape).view(np.uint8), ev.view(np.uint8)), case.name


# ---- chunked prefill ----------------------------------------------------
def tiny_prefill_cases():
    """Small prefill steps: fresh requests (no history), continuing ones,
    one new token, MHA/GQA/MQA, block sizes 1..16, fp32 and bf16."""
    specs = [
        dict(dtype=DTYPE_F32, Hq=4, Hkv=2, D=8, block_size=4, context_lens=[5, 9, 3], new_tokens=[5, 3, 1], seed=31),
        dict(dtype=DTYPE_BF16, Hq=4, Hkv=1, D=8, block_size=2, context_lens=[7, 4], new_tokens=[2, 4], seed=32),
        dict(dtype=DTYPE_F32, Hq=3, Hkv=3, D=4, block_size=1, context_lens=[6, 2], new_tokens=[6, 1], seed=33),
        dict(dtype=DTYPE_BF16, Hq=8, Hkv=2, D=16, block_size=16, context_lens=[17, 40], new_tokens=[17, 9],
             seed=34, pool="factor", pool_factor=1.5),
    ]
    return [synth.build_prefill_case(f"ptiny{i}", **sp) for i, sp in enumerate(specs)]


def prefill_brute_force(pc, k_cache, v_cache):
    """Plain-Python causal attention: new token j of request b at position
    L_b - n_b + j over positions 0..that position."""
    q = _f64(pc, pc.q)
    K = _f64(pc, k_cache)
    V = _f64(pc, v_cache)
    G = pc.Hq // pc.Hkv
    out = np.zeros((pc.T, pc.Hq, pc.D))
    for b in range(pc.B):
        L = int(pc.context_lens[b])
        q0, q1 = int(pc.query_start[b]), int(pc.query_start[b + 1])
        n = q1 - q0
        for j in range(n):
            pos = L - n + j
            rows = [(int(pc.block_tables[b][t // pc.block_size]), t % pc.block_size) for t in range(pos + 1)]
            for h in range(pc.Hq):
                g = h // G
                s_ = [pc.scale * sum(float(q[q0 + j, h, d]) * float(K[p_, o, g, d]) for d in range(pc.D))
                      for (p_, o) in rows]
                m = max(s_)
                w = [math.exp(x - m) for x in s_]
                tot = sum(w)
                for d in range(pc.D):
                    out[q0 + j, h, d] = sum(w[i] * float(V[p_, o, g, d]) for i, (p_, o) in enumerate(rows)) / tot
    return out


def pin_prefill_brute_force(orc):
    for pc in tiny_prefill_cases():
        kc, vc = orc.prefill_append(pc)
        np.testing.assert_allclose(orc.prefill(pc, kc, vc), prefill_brute_force(pc, kc, vc), rtol=1e-12,
                                   atol=1e-13, err_msg=pc.name)


def pin_prefill_one_token_is_decode(orc):
    """One new token per request: prefill is exactly the decode step."""
    for dc in tiny_cases() + [synth.make_config(1)]:
        kc, vc = orc.kv_append(dc)
        pc = synth.PagedPrefillCase(
            name=dc.name + "-as-prefill", dtype=dc.dtype, B=dc.B, T=dc.B, Hq=dc.Hq, Hkv=dc.Hkv, D=dc.D,
            block_size=dc.block_size, num_blocks=dc.num_blocks, max_blocks_per_seq=dc.max_blocks_per_seq,
            context_lens=dc.context_lens, query_start=np.arange(dc.B + 1, dtype=np.int32),
            block_tables=dc.block_tables, slot_mapping=dc.slot_mapping, q=dc.q, k_new=dc.k_new, v_new=dc.v_new,
            k_cache=kc, v_cache=vc, scale=dc.scale)
        assert np.array_equal(orc.prefill(pc, kc, vc), orc.decode(dc, kc, vc)), dc.name


def pin_prefill_fresh_first_token_is_v(orc):
    """A request with no history: its first new token sees only itself, so
    its output is its own V row, exactly."""
    for pc in tiny_prefill_cases():
        kc, vc = orc.prefill_append(pc)
        out = orc.prefill(pc, kc, vc)
        vnew = _f64(pc, pc.v_new)
        G = pc.Hq // pc.Hkv
        for b in range(pc.B):
            q0, q1 = int(pc.query_start[b]), int(pc.query_start[b + 1])
            if q1 - q0 != int(pc.context_lens[b]) or q1 == q0:
                continue
            for h in range(pc.Hq):
                assert np.array_equal(out[q0, h], vnew[q0, h // G]), (pc.name, b, h)


def pin_prefill_causal(orc):
    """Changing the K/V of a request's last new token changes only that
    token's output: no earlier token sees a later one."""
    for pc in tiny_prefill_cases():
        kc, vc = orc.prefill_append(pc)
        out = orc.prefill(pc, kc, vc)
        pos = pc.positions()
        for b in range(pc.B):
            q0, q1 = int(pc.query_start[b]), int(pc.query_start[b + 1])
            if q1 - q0 < 2:
                continue
            last = q1 - 1
            slot = int(pc.slot_mapping[last])
            k2, v2 = kc.copy(), vc.copy()
            blk, row = slot // pc.block_size, slot % pc.block_size
            if k2.dtype == np.uint16:                      # flip the sign of every value of that token
                k2[blk, row] ^= np.uint16(0x8000)
                v2[blk, row] ^= np.uint16(0x8000)
            else:
                k2[blk, row] = -k2[blk, row]
                v2[blk, row] = -v2[blk, row]
            out2 = orc.prefill(pc, k2, v2)
            assert np.array_equal(out[q0:last], out2[q0:last]), (pc.name, b, "earlier tokens changed")
            assert not np.array_equal(out[last], out2[last]), (pc.name, b, "the last token did not see itself")
            assert pos[last] == int(pc.context_lens[b]) - 1


ALL_PINS = [pin_golden_decode, pin_golden_append, pin_brute_force, pin_dense_numpy,
            pin_paged_equals_contiguous, pin_gqa_equals_repeated_mha, pin_block_permutation,
            pin_single_token_returns_v, pin_identical_keys_mean_v, pin_partitioned_equals_unsplit,
            pin_append_matches_index_assignment, pin_prefill_brute_force, pin_prefill_one_token_is_decode,
            pin_prefill_fresh_first_token_is_v, pin_prefill_causal]


if __name__ == "__main__":
    # Used by the mutant test: run every pin against the library given on the
    # command line and print the names of the pins that fail.
    import sys
    import oracle
    o = oracle.Oracle(sys.argv[1])
    failed = []
    for pin in ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError) as exc:  # ValueError: oracle rejected its input
            failed.append(pin.__name__)
    print(json.dumps(failed))
