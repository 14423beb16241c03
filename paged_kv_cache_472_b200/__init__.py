"""Python binding of libpagedattn (ctypes; argument marshalling only).

Every function here forwards to the C entry point of the same name declared
in include/pagedattn.h; all computation runs in the library's CUDA kernels.
Tensors may be torch tensors (their ``data_ptr()`` is passed) or raw integer
device pointers.  The library must be built (``build.build()``); importing
this package raises if ``libpagedattn.so`` is missing -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

from .build import LIB as _LIB_PATH

__all__ = ["PagedAttnError", "Shape", "Plan", "DTYPE_F32", "DTYPE_BF16", "DTYPE_F16", "SPLIT_BALANCED", "SPLIT_FIXED",
           "DEVERR_BLOCK_ID", "DEVERR_CONTEXT_LEN", "DEVERR_TIMEOUT", "DEVERR_WORKSPACE", "DEVERR_SLOT", "DEVERR_SMEM",
           "PLAN_NO_SPECULATION", "PLAN_TEST_MISGUESS", "PLAN_TEST_STALL", "pa_no_alloc_device_error",
           "pa_version", "pa_status_str", "pa_last_error_message", "pa_kv_append", "pa_plan",
           "pa_decode_workspace_size", "pa_workspace_init", "pa_decode", "pa_kv_append_decode", "pa_get_device_error",
           "pa_decode_no_alloc", "PrefillPlan", "pa_prefill_plan", "pa_prefill", "lib"]

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_WORKSPACE = range(5)
DTYPE_F32, DTYPE_BF16, DTYPE_F16 = 0, 1, 2
SPLIT_BALANCED, SPLIT_FIXED = 0, 1
DEVERR_BLOCK_ID, DEVERR_CONTEXT_LEN, DEVERR_TIMEOUT, DEVERR_WORKSPACE, DEVERR_SLOT, DEVERR_SMEM = (
    0x1, 0x2, 0x4, 0x8, 0x10, 0x20)
PLAN_NO_SPECULATION, PLAN_TEST_MISGUESS, PLAN_TEST_STALL = 0x1, 0x2, 0x4


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("dtype", ctypes.c_int32)]

    def __repr__(self):
        return "Shape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class Plan(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("partition_tokens", ctypes.c_int32), ("num_ctas", ctypes.c_int32),
                ("tile_tokens", ctypes.c_int32), ("stages", ctypes.c_int32), ("head_group", ctypes.c_int32),
                ("heads_per_unit", ctypes.c_int32), ("units_per_warp", ctypes.c_int32),
                ("warps_per_unit", ctypes.c_int32), ("max_context_len", ctypes.c_int32),
                ("smem_bytes", ctypes.c_int32), ("dynamic_share", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("split_merge", ctypes.c_int32), ("max_slots", ctypes.c_int64),
                ("shape", Shape), ("workspace_bytes", ctypes.c_size_t)]

    def as_dict(self):
        d = {n: getattr(self, n) for n, _ in self._fields_ if n != "shape"}
        d["shape"] = {n: getattr(self.shape, n) for n, _ in Shape._fields_}
        return d


class PrefillPlan(ctypes.Structure):
    _fields_ = [("q_tile", ctypes.c_int32), ("kv_tile", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("num_qtiles", ctypes.c_int32), ("max_new_tokens", ctypes.c_int32), ("smem_bytes", ctypes.c_int32),
                ("shape", Shape)]


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        self.status = status
        super().__init__(f"{where}: {pa_status_str(status)}: {message}")


if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libpagedattn.so is not built ({_LIB_PATH}); run paged_kv_cache_472_b200.build.build()")
lib = ctypes.CDLL(_LIB_PATH)

_vp, _i32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
_P = ctypes.POINTER
lib.pa_version.restype = _i32
lib.pa_status_str.argtypes = [ctypes.c_int]
lib.pa_status_str.restype = ctypes.c_char_p
lib.pa_last_error_message.restype = ctypes.c_char_p
lib.pa_kv_append.argtypes = [_vp, _vp, _vp, _vp, _vp, _P(Shape), _vp, _vp]
lib.pa_plan.argtypes = [_P(Shape), _i32, _i32, _i32, _P(Plan)]
lib.pa_decode_workspace_size.argtypes = [_P(Plan)]
lib.pa_decode_workspace_size.restype = _sz
lib.pa_workspace_init.argtypes = [_vp, _sz, _vp]
lib.pa_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _P(Shape), _P(Plan), _vp, _sz, _vp]
lib.pa_get_device_error.argtypes = [_vp, _i32, _P(_i32), _vp]
lib.pa_kv_append_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _P(Shape), _P(Plan),
                                    _vp, _sz, _vp]
lib.pa_decode_no_alloc.argtypes = [_vp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _P(Shape), _P(Plan), _vp]
lib.pa_no_alloc_device_error.argtypes = [_i32, _P(_i32), _vp]
lib.pa_prefill_plan.argtypes = [_P(Shape), _i32, _P(PrefillPlan)]
lib.pa_prefill.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _P(Shape), _P(PrefillPlan), _vp, _vp]
for _f in ("pa_kv_append", "pa_plan", "pa_workspace_init", "pa_decode", "pa_get_device_error",
           "pa_kv_append_decode", "pa_decode_no_alloc", "pa_no_alloc_device_error", "pa_prefill_plan", "pa_prefill"):
    getattr(lib, _f).restype = ctypes.c_int


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str):
    if st != PA_OK:
        raise PagedAttnError(st, where, lib.pa_last_error_message().decode())


def pa_version() -> int:
    return lib.pa_version()


def pa_status_str(status: int) -> str:
    return lib.pa_status_str(status).decode()


def pa_last_error_message() -> str:
    return lib.pa_last_error_message().decode()


def pa_kv_append(k_new, v_new, slot_mapping, k_cache, v_cache, shape: Shape, device_error=None, stream=None):
    _check(lib.pa_kv_append(_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache),
                            ctypes.byref(shape), _ptr(device_error), _stream(stream)), "pa_kv_append")


def pa_plan(shape: Shape, max_context_len: int, partition_tokens: int = 0, num_sms: int = 0) -> Plan:
    plan = Plan()
    _check(lib.pa_plan(ctypes.byref(shape), int(max_context_len), int(partition_tokens), int(num_sms),
                       ctypes.byref(plan)), "pa_plan")
    return plan


def pa_decode_workspace_size(plan: Plan) -> int:
    return lib.pa_decode_workspace_size(ctypes.byref(plan))


def pa_workspace_init(workspace, nbytes: int, stream=None):
    _check(lib.pa_workspace_init(_ptr(workspace), int(nbytes), _stream(stream)), "pa_workspace_init")


def pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, out, shape: Shape, plan: Plan,
              workspace, workspace_bytes: int, stream=None):
    _check(lib.pa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
                         float(scale), _ptr(out), ctypes.byref(shape), ctypes.byref(plan), _ptr(workspace),
                         int(workspace_bytes), _stream(stream)), "pa_decode")


def pa_kv_append_decode(k_new, v_new, slot_mapping, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                        out, shape: Shape, plan: Plan, workspace, workspace_bytes: int, stream=None):
    _check(lib.pa_kv_append_decode(_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), _ptr(q), _ptr(k_cache),
                                   _ptr(v_cache), _ptr(block_tables), _ptr(context_lens), float(scale), _ptr(out),
                                   ctypes.byref(shape), ctypes.byref(plan), _ptr(workspace), int(workspace_bytes),
                                   _stream(stream)), "pa_kv_append_decode")


def pa_decode_no_alloc(q, k_cache, v_cache, block_tables, context_lens, scale: float, out, shape: Shape, plan: Plan,
                       stream=None):
    _check(lib.pa_decode_no_alloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
                                  float(scale), _ptr(out), ctypes.byref(shape), ctypes.byref(plan), _stream(stream)),
           "pa_decode_no_alloc")


def pa_get_device_error(workspace, clear: bool = False, stream=None) -> int:
    err = _i32(0)
    _check(lib.pa_get_device_error(_ptr(workspace), int(bool(clear)), ctypes.byref(err), _stream(stream)),
           "pa_get_device_error")
    return err.value


def pa_no_alloc_device_error(clear: bool = False, stream=None) -> int:
    err = _i32(0)
    _check(lib.pa_no_alloc_device_error(int(bool(clear)), ctypes.byref(err), _stream(stream)),
           "pa_no_alloc_device_error")
    return err.value


def pa_prefill_plan(shape: Shape, max_new_tokens: int) -> PrefillPlan:
    plan = PrefillPlan()
    _check(lib.pa_prefill_plan(ctypes.byref(shape), max_new_tokens, ctypes.byref(plan)), "pa_prefill_plan")
    return plan


def pa_prefill(q, k_cache, v_cache, block_tables, context_lens, query_start, scale, out, shape: Shape,
               plan: PrefillPlan, device_error=None, stream=None):
    _check(lib.pa_prefill(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
                          _ptr(query_start), ctypes.c_float(scale), _ptr(out), ctypes.byref(shape),
                          ctypes.byref(plan), _ptr(device_error), _stream(stream)), "pa_prefill")
