"""Seeded synthetic inputs for paged decode attention and the KV append.

This module only *builds inputs*: request lengths, a physical block pool with a
free-list allocation, block tables, the append slot of each request, and the
q / K / V values.  It holds none of the attention arithmetic, so both the
float64 oracle and the CUDA library can be fed from it without sharing any
part of what they compute.

Layouts follow the paged storage described on the BareLLM page ("Paged KV
cache" and "Cache layers": K/V tensors shaped
``[physical_blocks, block_size, kv_heads, head_dim]`` in token-before-head
(NHD) order, one layer per call) and the Nano-vLLM page ("Kernmodul:
Sequence": a block table per sequence).

Workloads (one per decode batch shape; ``make_config(i)``):
  1. tiny fp32: B=2, L={17,33}, Hq=4, Hkv=2, D=64, bs=16, pool of 8 blocks
  2. Qwen3-0.6B-shaped bf16: B=32, 16/8/128, bs=16, L ~ U[128,2048]
  3. Llama-3.2-1B-shaped bf16: B=128, 32/8/64, bs=16, L ~ U[512,4096],
     pool 1.5x the blocks needed, random free-list order
  4. long-context MQA bf16: B=8, 32/1/128, bs=256, L ~ U[32768,131072],
     fixed 512-token partitions
  5. Qwen3-8B-shaped mixed bf16: B=256, 32/8/128, bs=16, log-normal lengths
     (median 1024, sigma 1) clipped to [16,16384]; requests 8k..8k+7 share
     their first full prefix blocks (at most 4)

Conventions (the pages leave these open; the readings are stated here):
  * ``context_lens[b]`` counts the token being appended this step, so the
    append slot is position ``L_b - 1`` and decode attends to it.
  * ``slot_mapping[b] = phys * block_size + offset`` (int32, < 0 = skip).
  * block-table entries past ``ceil(L_b / bs)`` are -1 and never read.
  * lengths, pool order and tables come from numpy's PCG64 seeded with
    ``1000 + config id``; q, k, v ~ N(0, 1) come from a counter-based
    Philox4x32-10 + Box-Muller generator (``normals.c``) keyed by a seed drawn
    from that stream, rounded to bf16 (nearest-even) on the CPU for bf16
    cases, so every consumer reads identical bits.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_GEN_SRC = os.path.join(_HERE, "normals.c")
_GEN_LIB = os.path.join(_HERE, "libsynthnormals.so")
_gen = None


def build(force: bool = False) -> str:
    """Compile the counter-based normal generator (gcc, OpenMP)."""
    if force or not os.path.exists(_GEN_LIB) or os.path.getmtime(_GEN_LIB) < os.path.getmtime(_GEN_SRC):
        subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", _GEN_LIB,
                        _GEN_SRC, "-lm"], check=True)
    return _GEN_LIB


def _lib():
    global _gen
    if _gen is None:
        lib = ctypes.CDLL(build())
        lib.synth_normals.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64,
                                      ctypes.c_void_p, ctypes.c_void_p]
        lib.synth_normals.restype = None
        lib.synth_philox4x32_10.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.synth_philox4x32_10.restype = None
        _gen = lib
    return _gen


def philox4x32_10(ctr, key) -> np.ndarray:
    """One Philox4x32-10 block (exposed for its known-answer test)."""
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    _lib().synth_philox4x32_10(c.ctypes.data, k.ctypes.data, out.ctypes.data)
    return out


def normals(seed: int, stream: int, shape, dtype: str) -> np.ndarray:
    """N(0,1) values of the given shape: float32, or bf16 / fp16 bit patterns (uint16)."""
    n = int(np.prod(shape))
    if dtype in (DTYPE_F32, DTYPE_F16):
        out = np.empty(n, dtype=np.float32)
        _lib().synth_normals(seed, stream, n, out.ctypes.data, None)
        if dtype == DTYPE_F16:  # nearest-even, as numpy's float32 -> float16 cast
            out = out.astype(np.float16).view(np.uint16)
    else:
        out = np.empty(n, dtype=np.uint16)
        _lib().synth_normals(seed, stream, n, None, out.ctypes.data)
    return out.reshape(shape)

DTYPE_F32 = "f32"
DTYPE_BF16 = "bf16"
DTYPE_F16 = "f16"


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the
    16-bit patterns as uint16.  Inputs here are finite normals, so NaN/Inf
    need no special case."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32 exactly."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class PagedDecodeCase:
    """One decode step's inputs.  Arrays are host numpy arrays.

    For ``dtype == 'bf16'`` the value arrays hold uint16 bit patterns; for
    ``'f32'`` they hold float32.  ``k_cache``/``v_cache`` are the pool
    contents *before* the append of this step.
    """
    name: str
    dtype: str
    B: int
    Hq: int
    Hkv: int
    D: int
    block_size: int
    num_blocks: int
    max_blocks_per_seq: int
    context_lens: np.ndarray      # [B] int32
    block_tables: np.ndarray      # [B, max_blocks_per_seq] int32, -1 = unused
    slot_mapping: np.ndarray      # [B] int32
    q: np.ndarray                 # [B, Hq, D]
    k_new: np.ndarray             # [B, Hkv, D]
    v_new: np.ndarray             # [B, Hkv, D]
    k_cache: np.ndarray           # [num_blocks, block_size, Hkv, D]
    v_cache: np.ndarray           # [num_blocks, block_size, Hkv, D]
    scale: float
    partition_tokens: int = 0     # 0 = let the planner choose
    seed: int = 0
    notes: dict = field(default_factory=dict)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == DTYPE_F32 else 2

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    def as_float32(self, a: np.ndarray) -> np.ndarray:
        """Value array widened to float32 (exact for every dtype)."""
        if self.dtype == DTYPE_BF16:
            return bf16_bits_to_f32(a)
        if self.dtype == DTYPE_F16:
            return np.asarray(a, np.uint16).view(np.float16).astype(np.float32)
        return np.asarray(a, np.float32)

    def blocks_used(self) -> int:
        return int(sum(-(-int(L) // self.block_size) for L in self.context_lens))

    def kv_bytes_logical(self) -> int:
        """K+V bytes a decode step reads, counting each request's own reads."""
        return int(self.context_lens.astype(np.int64).sum()) * self.Hkv * self.D * self.elem_bytes * 2

    def kv_bytes_unique(self) -> int:
        """K+V bytes a decode step must read at least: every physical block
        once, as many of its rows as the request reading most of it reads
        (prefix blocks that several tables name are counted once)."""
        rows = {}
        for b in range(self.B):
            L = int(self.context_lens[b])
            for j in range(-(-L // self.block_size)):
                blk = int(self.block_tables[b, j])
                rows[blk] = max(rows.get(blk, 0), min(self.block_size, L - j * self.block_size))
        return sum(rows.values()) * self.Hkv * self.D * self.elem_bytes * 2

    def unique_blocks(self) -> int:
        ids = set()
        for b in range(self.B):
            n = -(-int(self.context_lens[b]) // self.block_size)
            ids.update(int(x) for x in self.block_tables[b, :n])
        return len(ids)


_STREAM_Q, _STREAM_KNEW, _STREAM_VNEW, _STREAM_KCACHE, _STREAM_VCACHE = range(5)


def build_case(name: str, *, dtype: str, Hq: int, Hkv: int, D: int, block_size: int,
               context_lens, seed: int, pool: str = "exact", pool_factor: float = 1.0,
               share_group: int = 0, share_max_blocks: int = 0, max_blocks_per_seq: int | None = None,
               extra_blocks: int = 0, partition_tokens: int = 0, values: bool = True) -> PagedDecodeCase:
    """Build one seeded decode step.

    pool="exact": the pool holds exactly the blocks the batch uses (plus
    ``extra_blocks``) and they are handed out in a seeded random order.
    pool="factor": the pool holds ceil(pool_factor * blocks needed) blocks;
    a seeded permutation of all ids is the free list, popped request by
    request, position by position.
    share_group=g>0: requests g*k .. g*k+g-1 reference the same physical
    blocks for their first min(share_max_blocks, floor((L_b-1)/bs)) blocks
    (full blocks wholly before the append position, as prefix caching
    reuses full blocks).
    """
    rng = np.random.default_rng(seed)
    lens = np.asarray(context_lens, dtype=np.int64)
    B = int(lens.shape[0])
    bs = block_size
    nblk = [-(-int(L) // bs) for L in lens]
    if max_blocks_per_seq is None:
        max_blocks_per_seq = max(max(nblk), 1)
    assert max_blocks_per_seq >= max(nblk)

    # Which leading blocks of each request are shared with its group.
    n_shared = [0] * B
    group_shared = {}
    if share_group > 0:
        for b in range(B):
            n_shared[b] = min(share_max_blocks, max((int(lens[b]) - 1) // bs, 0))
        for gk in range(0, B, share_group):
            members = range(gk, min(gk + share_group, B))
            group_shared[gk] = max(n_shared[b] for b in members)
    needed = sum(nblk) - sum(n_shared) + sum(group_shared.values())

    if pool == "exact":
        num_blocks = needed + extra_blocks
    elif pool == "factor":
        num_blocks = int(math.ceil(pool_factor * needed))
    else:
        raise ValueError(pool)
    free_list = list(rng.permutation(num_blocks).astype(np.int64))
    free_list.reverse()  # pop() from the end == take the permutation front to back

    tables = np.full((B, max_blocks_per_seq), -1, dtype=np.int32)
    group_ids = {}
    for b in range(B):
        if share_group > 0:
            gk = (b // share_group) * share_group
            if gk not in group_ids:
                group_ids[gk] = [free_list.pop() for _ in range(group_shared[gk])]
            for j in range(n_shared[b]):
                tables[b, j] = group_ids[gk][j]
        for j in range(n_shared[b], nblk[b]):
            tables[b, j] = free_list.pop()

    slots = np.empty(B, dtype=np.int32)
    for b in range(B):
        pos = int(lens[b]) - 1
        slots[b] = int(tables[b, pos // bs]) * bs + pos % bs if pos >= 0 else -1

    if values:
        vseed = int(rng.integers(0, 2**63 - 1))
        q = normals(vseed, _STREAM_Q, (B, Hq, D), dtype)
        k_new = normals(vseed, _STREAM_KNEW, (B, Hkv, D), dtype)
        v_new = normals(vseed, _STREAM_VNEW, (B, Hkv, D), dtype)
        k_cache = normals(vseed, _STREAM_KCACHE, (num_blocks, bs, Hkv, D), dtype)
        v_cache = normals(vseed, _STREAM_VCACHE, (num_blocks, bs, Hkv, D), dtype)
    else:
        shp = lambda *s: np.zeros(s, dtype=np.float32 if dtype == DTYPE_F32 else np.uint16)
        q, k_new, v_new = shp(B, Hq, D), shp(B, Hkv, D), shp(B, Hkv, D)
        k_cache, v_cache = shp(num_blocks, bs, Hkv, D), shp(num_blocks, bs, Hkv, D)

    return PagedDecodeCase(
        name=name, dtype=dtype, B=B, Hq=Hq, Hkv=Hkv, D=D, block_size=bs, num_blocks=num_blocks,
        max_blocks_per_seq=max_blocks_per_seq, context_lens=lens.astype(np.int32), block_tables=tables,
        slot_mapping=slots, q=q, k_new=k_new, v_new=v_new, k_cache=k_cache, v_cache=v_cache,
        scale=1.0 / math.sqrt(D), partition_tokens=partition_tokens, seed=seed,
        notes={"pool": pool, "pool_factor": pool_factor, "share_group": share_group})


# ----------------------------------------------------------------------------
# The five decode batch shapes.
# ----------------------------------------------------------------------------
CONFIG_NAMES = {
    1: "tiny-fp32-gqa2-d64",
    2: "qwen3-0.6b-decode-b32",
    3: "llama-3.2-1b-decode-b128",
    4: "long-mqa-splitk-b8",
    5: "qwen3-8b-mixed-b256",
}
LOGNORMAL_SIGMA = 1.0


def config_lengths(cid: int, rng: np.random.Generator, batch: int | None = None) -> np.ndarray:
    """Context lengths of workload ``cid`` (integers; uniform ranges inclusive)."""
    if cid == 1:
        return np.array([17, 33], dtype=np.int64)
    if cid == 2:
        return rng.integers(128, 2048, size=batch or 32, endpoint=True)
    if cid == 3:
        return rng.integers(512, 4096, size=batch or 128, endpoint=True)
    if cid == 4:
        return rng.integers(32768, 131072, size=batch or 8, endpoint=True)
    if cid == 5:
        x = rng.lognormal(mean=math.log(1024.0), sigma=LOGNORMAL_SIGMA, size=batch or 256)
        return np.clip(np.rint(x), 16, 16384).astype(np.int64)
    raise ValueError(cid)


def make_config(cid: int, seed: int | None = None, batch: int | None = None,
                values: bool = True) -> PagedDecodeCase:
    """Workload ``cid`` (1..5) with seed ``1000 + cid`` unless given.

    ``batch`` overrides B (a smaller batch of the same length distribution,
    used where the full batch would be too slow for the float64 oracle).
    """
    seed = 1000 + cid if seed is None else seed
    rng = np.random.default_rng(seed)
    lens = config_lengths(cid, rng, batch)
    sub = int(rng.integers(0, 2**31 - 1))
    name = CONFIG_NAMES[cid] + ("" if batch is None else f"-subset{batch}")
    if cid == 1:
        c = build_case(name, dtype=DTYPE_F32, Hq=4, Hkv=2, D=64, block_size=16, context_lens=lens,
                       seed=sub, pool="exact", extra_blocks=3, values=values)
        return c
    if cid == 2:
        return build_case(name, dtype=DTYPE_BF16, Hq=16, Hkv=8, D=128, block_size=16,
                          context_lens=lens, seed=sub, pool="exact", max_blocks_per_seq=2048 // 16,
                          values=values)
    if cid == 3:
        return build_case(name, dtype=DTYPE_BF16, Hq=32, Hkv=8, D=64, block_size=16,
                          context_lens=lens, seed=sub, pool="factor", pool_factor=1.5,
                          max_blocks_per_seq=4096 // 16, values=values)
    if cid == 4:
        return build_case(name, dtype=DTYPE_BF16, Hq=32, Hkv=1, D=128, block_size=256,
                          context_lens=lens, seed=sub, pool="exact", max_blocks_per_seq=131072 // 256,
                          partition_tokens=512, values=values)
    if cid == 5:
        return build_case(name, dtype=DTYPE_BF16, Hq=32, Hkv=8, D=128, block_size=16,
                          context_lens=lens, seed=sub, pool="exact", share_group=8, share_max_blocks=4,
                          max_blocks_per_seq=16384 // 16, values=values)
    raise ValueError(cid)


# ----------------------------------------------------------------------------
# Chunked prefill: several new tokens per request.
# ----------------------------------------------------------------------------
@dataclass
class PagedPrefillCase:
    """One chunked-prefill step's inputs (host numpy arrays, value arrays as in
    PagedDecodeCase).  Request b owns rows query_start[b] .. query_start[b+1]-1
    of q / k_new / v_new / slot_mapping: its n_b new tokens, the last n_b of
    its context_lens[b] positions.  ``k_cache``/``v_cache`` hold the history
    (and stale values at the new tokens' slots, overwritten by the append)."""
    name: str
    dtype: str
    B: int
    T: int
    Hq: int
    Hkv: int
    D: int
    block_size: int
    num_blocks: int
    max_blocks_per_seq: int
    context_lens: np.ndarray      # [B] int32, history + new tokens
    query_start: np.ndarray       # [B + 1] int32
    block_tables: np.ndarray      # [B, max_blocks_per_seq] int32
    slot_mapping: np.ndarray      # [T] int32
    q: np.ndarray                 # [T, Hq, D]
    k_new: np.ndarray             # [T, Hkv, D]
    v_new: np.ndarray             # [T, Hkv, D]
    k_cache: np.ndarray
    v_cache: np.ndarray
    scale: float
    seed: int = 0
    notes: dict = field(default_factory=dict)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == DTYPE_F32 else 2

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    def as_float32(self, a: np.ndarray) -> np.ndarray:
        if self.dtype == DTYPE_BF16:
            return bf16_bits_to_f32(a)
        if self.dtype == DTYPE_F16:
            return np.asarray(a, np.uint16).view(np.float16).astype(np.float32)
        return np.asarray(a, np.float32)

    def new_tokens(self) -> np.ndarray:
        return np.diff(self.query_start.astype(np.int64))

    def positions(self) -> np.ndarray:
        """[T] position of every new token in its request's context."""
        pos = np.empty(self.T, dtype=np.int64)
        for b in range(self.B):
            q0, q1 = int(self.query_start[b]), int(self.query_start[b + 1])
            pos[q0:q1] = int(self.context_lens[b]) - (q1 - q0) + np.arange(q1 - q0)
        return pos

    def visible_pairs(self) -> int:
        """(query token, key position) pairs the causal prefill computes."""
        return int((self.positions() + 1).sum())


_STREAM_PQ, _STREAM_PKNEW, _STREAM_PVNEW = 5, 6, 7


def build_prefill_case(name: str, *, dtype: str, Hq: int, Hkv: int, D: int, block_size: int, context_lens,
                       new_tokens, seed: int, values: bool = True, **pool) -> PagedPrefillCase:
    """A seeded prefill step: the pool, tables and history as build_case makes
    them for ``context_lens`` (history + new tokens), the new tokens' slots,
    and q / new K / new V for every new token."""
    lens = np.asarray(context_lens, dtype=np.int64)
    n = np.asarray(new_tokens, dtype=np.int64)
    assert lens.shape == n.shape and np.all(n >= 0) and np.all(n <= lens)
    base = build_case(name, dtype=dtype, Hq=Hq, Hkv=Hkv, D=D, block_size=block_size, context_lens=lens,
                      seed=seed, values=values, **pool)
    B, bs = base.B, block_size
    qs = np.zeros(B + 1, dtype=np.int32)
    qs[1:] = np.cumsum(n)
    T = int(qs[-1])
    slots = np.empty(T, dtype=np.int32)
    for b in range(B):
        for j in range(int(n[b])):
            pos = int(lens[b]) - int(n[b]) + j
            slots[qs[b] + j] = int(base.block_tables[b, pos // bs]) * bs + pos % bs
    if values:
        vseed = int(np.random.default_rng(seed ^ 0x5DEECE66D).integers(0, 2**63 - 1))
        q = normals(vseed, _STREAM_PQ, (T, Hq, D), dtype)
        k_new = normals(vseed, _STREAM_PKNEW, (T, Hkv, D), dtype)
        v_new = normals(vseed, _STREAM_PVNEW, (T, Hkv, D), dtype)
    else:
        shp = lambda *s_: np.zeros(s_, dtype=np.float32 if dtype == DTYPE_F32 else np.uint16)
        q, k_new, v_new = shp(T, Hq, D), shp(T, Hkv, D), shp(T, Hkv, D)
    return PagedPrefillCase(name=name, dtype=dtype, B=B, T=T, Hq=Hq, Hkv=Hkv, D=D, block_size=bs,
                            num_blocks=base.num_blocks, max_blocks_per_seq=base.max_blocks_per_seq,
                            context_lens=base.context_lens, query_start=qs, block_tables=base.block_tables,
                            slot_mapping=slots, q=q, k_new=k_new, v_new=v_new, k_cache=base.k_cache,
                            v_cache=base.v_cache, scale=1.0 / math.sqrt(D), seed=seed, notes=base.notes)


PREFILL_NAMES = {
    1: "qwen3-8b-prefill-chunk512-b8",
    2: "llama-3.2-1b-prefill-mixed-b16",
}


def make_prefill_config(pid: int, seed: int | None = None, batch: int | None = None, chunk: int | None = None,
                        values: bool = True) -> PagedPrefillCase:
    """Chunked-prefill workloads (seed 2000 + pid unless given):
      1. Qwen3-8B-shaped chunk: B=8, 32/8/128, bs=16, history ~ U[0, 3584],
         512 new tokens per request (a 4096-token chunk);
      2. Llama-3.2-1B-shaped mixed: B=16, 32/8/64, bs=16, history ~ U[0, 2048],
         new tokens ~ U[1, 512] (some requests fresh, some continuing).
    ``batch`` / ``chunk`` shrink the batch / the new tokens per request."""
    seed = 2000 + pid if seed is None else seed
    rng = np.random.default_rng(seed)
    sub = int(rng.integers(0, 2**31 - 1))
    name = PREFILL_NAMES[pid] + ("" if batch is None and chunk is None else f"-subset{batch}x{chunk}")
    if pid == 1:
        B = batch or 8
        n = np.full(B, chunk or 512, dtype=np.int64)
        hist = rng.integers(0, 3584, size=B, endpoint=True)
        return build_prefill_case(name, dtype=DTYPE_BF16, Hq=32, Hkv=8, D=128, block_size=16,
                                  context_lens=hist + n, new_tokens=n, seed=sub, values=values, pool="exact")
    if pid == 2:
        B = batch or 16
        n = rng.integers(1, chunk or 512, size=B, endpoint=True)
        hist = rng.integers(0, 2048, size=B, endpoint=True)
        hist[::4] = 0  # every fourth request starts fresh
        return build_prefill_case(name, dtype=DTYPE_BF16, Hq=32, Hkv=8, D=64, block_size=16,
                                  context_lens=hist + n, new_tokens=n, seed=sub, values=values,
                                  pool="factor", pool_factor=1.25)
    raise ValueError(pid)


def prefill_algorithmic(pc: PagedPrefillCase) -> dict:
    """Flops of the causal prefill (QK^T and PV over the visible pairs) and
    the bytes it must move at least (each request's K/V once, q in, out)."""
    e = pc.elem_bytes
    flops = 4 * pc.visible_pairs() * pc.Hq * pc.D
    kv = int(pc.context_lens.astype(np.int64).sum()) * pc.Hkv * pc.D * e * 2
    qo = 2 * pc.T * pc.Hq * pc.D * e
    return {"flops": flops, "bytes": kv + qo}


def algorithmic_bytes(case: PagedDecodeCase) -> dict:
    """Bytes one decode step must move: K+V each request reads, q in, out
    written, block-table entries and lengths read (``decode_total``, each
    request's own reads; ``decode_unique``, a block several requests share
    counted once).  Append bytes (read k_new/v_new, write the slot) are
    listed separately."""
    e = case.elem_bytes
    kv = case.kv_bytes_logical()
    qo = 2 * case.B * case.Hq * case.D * e
    tables = 4 * case.blocks_used() + 4 * case.B
    append = 4 * case.B * case.Hkv * case.D * e + 4 * case.B
    unique_kv = case.kv_bytes_unique()
    return {"kv": kv, "q_out": qo, "tables": tables, "decode_total": kv + qo + tables,
            "append": append, "step_total": kv + qo + tables + append, "kv_unique": unique_kv,
            "decode_unique": unique_kv + qo + tables}
