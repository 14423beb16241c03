"""Float64 CPU oracle for paged decode attention and the KV append.

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and the
CPU baseline / reference leg of ``bench.py`` may import this package.  The
library under test never does, and nothing here imports the library: the two
share only the seeded input generator in ``synth``.

The arithmetic lives in ``paged_attn_oracle.c`` (plain C, double precision);
this module is the ctypes marshalling around it plus its build step.
Pinned by ``tests/test_oracle.py`` (invariants, closed forms, brute force,
hand-derived fixtures in ``tests/golden`` and planted mistakes).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "paged_attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB, extra_flags=()) -> str:
    """Compile the oracle with gcc (no FMA contraction, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", *CFLAGS, *extra_flags, "-o", out, src, "-lm"]
        subprocess.run(cmd, check=True)
    return out


class _Problem(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("block_tables", ctypes.c_void_p), ("context_lens", ctypes.c_void_p),
        ("scale", ctypes.c_double),
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32),
        ("block_size", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32), ("dtype", ctypes.c_int32),
    ]


class Oracle:
    """ctypes view of one compiled oracle library (the real one, or a test's
    deliberately broken copy)."""

    def __init__(self, path: str | None = None):
        self.path = path or build()
        lib = ctypes.CDLL(self.path)
        vp, i32 = ctypes.c_void_p, ctypes.c_int
        pp = ctypes.POINTER(_Problem)
        lib.oracle_decode.argtypes = [pp, vp, i32]
        lib.oracle_decode_pairs.argtypes = [pp, vp, i32, vp, i32]
        lib.oracle_decode_partitioned.argtypes = [pp, i32, vp, i32]
        lib.oracle_kv_append.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32]
        lib.oracle_prefill.argtypes = [pp, vp, vp, i32]
        lib.oracle_prefill_rows.argtypes = [pp, vp, vp, i32, vp, i32]
        for f in (lib.oracle_decode, lib.oracle_decode_pairs, lib.oracle_decode_partitioned,
                  lib.oracle_kv_append, lib.oracle_max_threads, lib.oracle_prefill, lib.oracle_prefill_rows):
            f.restype = ctypes.c_int
        self.lib = lib

    # -- helpers ---------------------------------------------------------
    @staticmethod
    def _dtype_code(dtype: str) -> int:
        return {"f32": 0, "bf16": 1, "f16": 2}[dtype]

    @staticmethod
    def _c(a: np.ndarray, dt) -> np.ndarray:
        return np.ascontiguousarray(a, dtype=dt)

    def _problem(self, case, q, k_cache, v_cache, block_tables=None, context_lens=None):
        vdt = np.float32 if case.dtype == "f32" else np.uint16
        keep = [self._c(q, vdt), self._c(k_cache, vdt), self._c(v_cache, vdt),
                self._c(case.block_tables if block_tables is None else block_tables, np.int32),
                self._c(case.context_lens if context_lens is None else context_lens, np.int32)]
        p = _Problem(keep[0].ctypes.data, keep[1].ctypes.data, keep[2].ctypes.data,
                     keep[3].ctypes.data, keep[4].ctypes.data, float(case.scale),
                     case.B, case.Hq, case.Hkv, case.D, case.block_size, keep[1].shape[0],
                     keep[3].shape[1], self._dtype_code(case.dtype))
        return p, keep

    # -- the oracle's entry points ---------------------------------------
    def max_threads(self) -> int:
        return self.lib.oracle_max_threads()

    def kv_append(self, case, k_cache=None, v_cache=None):
        """Return (k_cache, v_cache) after the append (fresh copies)."""
        vdt = np.float32 if case.dtype == "f32" else np.uint16
        kc = np.array(case.k_cache if k_cache is None else k_cache, dtype=vdt, copy=True)
        vc = np.array(case.v_cache if v_cache is None else v_cache, dtype=vdt, copy=True)
        kn, vn = self._c(case.k_new, vdt), self._c(case.v_new, vdt)
        sm = self._c(case.slot_mapping, np.int32)
        rc = self.lib.oracle_kv_append(kn.ctypes.data, vn.ctypes.data, sm.ctypes.data, kc.ctypes.data,
                                       vc.ctypes.data, case.B, case.Hkv, case.D, case.block_size,
                                       kc.shape[0], self._dtype_code(case.dtype))
        if rc < 0:
            raise ValueError(f"oracle_kv_append rejected the input ({rc})")
        return kc, vc

    def decode(self, case, k_cache=None, v_cache=None, *, q=None, block_tables=None, context_lens=None,
               nthreads: int = 0) -> np.ndarray:
        """out[B, Hq, D] (float64) over the given pool (default: the case's
        pool after its append)."""
        if k_cache is None or v_cache is None:
            k_cache, v_cache = self.kv_append(case)
        p, keep = self._problem(case, case.q if q is None else q, k_cache, v_cache, block_tables,
                                context_lens)
        out = np.zeros((case.B, case.Hq, case.D), dtype=np.float64)
        rc = self.lib.oracle_decode(ctypes.byref(p), out.ctypes.data, nthreads)
        if rc:
            raise ValueError(f"oracle_decode rejected the input ({rc})")
        return out

    def decode_pairs(self, case, pairs, k_cache=None, v_cache=None, nthreads: int = 0) -> np.ndarray:
        """out[len(pairs), D] for the listed (request, query head) pairs."""
        if k_cache is None or v_cache is None:
            k_cache, v_cache = self.kv_append(case)
        p, keep = self._problem(case, case.q, k_cache, v_cache)
        pr = self._c(np.asarray(pairs).reshape(-1, 2), np.int32)
        out = np.zeros((pr.shape[0], case.D), dtype=np.float64)
        rc = self.lib.oracle_decode_pairs(ctypes.byref(p), pr.ctypes.data, pr.shape[0], out.ctypes.data,
                                          nthreads)
        if rc:
            raise ValueError(f"oracle_decode_pairs rejected the input ({rc})")
        return out

    def decode_partitioned(self, case, partition_tokens: int, k_cache=None, v_cache=None,
                           nthreads: int = 0) -> np.ndarray:
        if k_cache is None or v_cache is None:
            k_cache, v_cache = self.kv_append(case)
        p, keep = self._problem(case, case.q, k_cache, v_cache)
        out = np.zeros((case.B, case.Hq, case.D), dtype=np.float64)
        rc = self.lib.oracle_decode_partitioned(ctypes.byref(p), partition_tokens, out.ctypes.data, nthreads)
        if rc:
            raise ValueError(f"oracle_decode_partitioned rejected the input ({rc})")
        return out


    # -- chunked prefill ---------------------------------------------------
    def prefill_append(self, pcase, k_cache=None, v_cache=None):
        """(k_cache, v_cache) after writing every new token's K/V to its slot."""
        vdt = np.float32 if pcase.dtype == "f32" else np.uint16
        kc = np.array(pcase.k_cache if k_cache is None else k_cache, dtype=vdt, copy=True)
        vc = np.array(pcase.v_cache if v_cache is None else v_cache, dtype=vdt, copy=True)
        kn, vn = self._c(pcase.k_new, vdt), self._c(pcase.v_new, vdt)
        sm = self._c(pcase.slot_mapping, np.int32)
        rc = self.lib.oracle_kv_append(kn.ctypes.data, vn.ctypes.data, sm.ctypes.data, kc.ctypes.data,
                                       vc.ctypes.data, pcase.T, pcase.Hkv, pcase.D, pcase.block_size,
                                       kc.shape[0], self._dtype_code(pcase.dtype))
        if rc < 0:
            raise ValueError(f"oracle_kv_append rejected the input ({rc})")
        return kc, vc

    def prefill(self, pcase, k_cache=None, v_cache=None, *, q=None, nthreads: int = 0) -> np.ndarray:
        """out[T, Hq, D] (float64) of the chunked prefill over the given pool
        (default: the case's pool after its new tokens are written)."""
        if k_cache is None or v_cache is None:
            k_cache, v_cache = self.prefill_append(pcase)
        p, keep = self._problem(pcase, pcase.q if q is None else q, k_cache, v_cache)
        qs = self._c(pcase.query_start, np.int32)
        out = np.zeros((pcase.T, pcase.Hq, pcase.D), dtype=np.float64)
        rc = self.lib.oracle_prefill(ctypes.byref(p), qs.ctypes.data, out.ctypes.data, nthreads)
        if rc:
            raise ValueError(f"oracle_prefill rejected the input ({rc})")
        return out

    def prefill_rows(self, pcase, rows, k_cache=None, v_cache=None, nthreads: int = 0) -> np.ndarray:
        """out[len(rows), Hq, D] of the prefill for the listed q rows only."""
        if k_cache is None or v_cache is None:
            k_cache, v_cache = self.prefill_append(pcase)
        p, keep = self._problem(pcase, pcase.q, k_cache, v_cache)
        qs = self._c(pcase.query_start, np.int32)
        r = self._c(np.asarray(rows).reshape(-1), np.int64)
        out = np.zeros((r.shape[0], pcase.Hq, pcase.D), dtype=np.float64)
        rc = self.lib.oracle_prefill_rows(ctypes.byref(p), qs.ctypes.data, r.ctypes.data, r.shape[0],
                                          out.ctypes.data, nthreads)
        if rc:
            raise ValueError(f"oracle_prefill_rows rejected the input ({rc})")
        return out


_DEFAULT: Oracle | None = None


def default() -> Oracle:
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT
