"""Torch plumbing around the C ABI: shapes from tensors, a planned decode with
its workspace allocated through torch, and dtype names.  No attention
arithmetic happens here; every compute step is a library call."""
from __future__ import annotations

import torch

from . import (DTYPE_BF16, DTYPE_F16, DTYPE_F32, Plan, Shape, pa_decode, pa_get_device_error, pa_kv_append,
               pa_kv_append_decode, pa_plan, pa_workspace_init)

TORCH_DTYPE = {DTYPE_F32: torch.float32, DTYPE_BF16: torch.bfloat16, DTYPE_F16: torch.float16}
PA_DTYPE = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16}


def shape_of(q: torch.Tensor, k_cache: torch.Tensor, block_tables: torch.Tensor) -> Shape:
    """Shape from q [B,Hq,D], k_cache [num_blocks,bs,Hkv,D], tables [B,max_blocks]."""
    B, Hq, D = q.shape
    nb, bs, Hkv, D2 = k_cache.shape
    assert D == D2 and q.dtype == k_cache.dtype
    return Shape(B, Hq, Hkv, D, bs, nb, block_tables.shape[1], PA_DTYPE[q.dtype])


class PagedDecoder:
    """A plan plus a workspace for one decode shape on one device.

    ``partition_tokens`` 0 = balanced split; > 0 = fixed partitions.
    ``max_context_len`` sizes the fixed-partition workspace.
    """

    def __init__(self, shape: Shape, max_context_len: int, partition_tokens: int = 0, num_sms: int = 0,
                 device: torch.device | str = "cuda"):
        self.shape = shape
        self.plan: Plan = pa_plan(shape, max_context_len, partition_tokens, num_sms)
        self.workspace_bytes = int(self.plan.workspace_bytes)
        # 256-byte aligned (the caching allocator hands out 512-byte aligned blocks)
        self.workspace = torch.empty(max(self.workspace_bytes, 256), dtype=torch.uint8, device=device)
        pa_workspace_init(self.workspace, self.workspace.numel())

    def decode(self, q, k_cache, v_cache, block_tables, context_lens, scale, out, stream=None):
        pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, self.shape, self.plan,
                  self.workspace, self.workspace.numel(), stream)
        return out

    def append(self, k_new, v_new, slot_mapping, k_cache, v_cache, stream=None):
        pa_kv_append(k_new, v_new, slot_mapping, k_cache, v_cache, self.shape, self.workspace, stream)

    def append_decode(self, k_new, v_new, slot_mapping, q, k_cache, v_cache, block_tables, context_lens, scale, out,
                      stream=None):
        pa_kv_append_decode(k_new, v_new, slot_mapping, q, k_cache, v_cache, block_tables, context_lens, scale, out,
                            self.shape, self.plan, self.workspace, self.workspace.numel(), stream)
        return out

    def device_error(self, clear: bool = False) -> int:
        return pa_get_device_error(self.workspace, clear)


class StepStaging:
    """One decode step's per-step inputs (q, new K/V, slot mapping, context
    lengths, block tables) packed in one pinned host buffer and one device
    buffer, so a step uploads them with a single copy.  Each named view is a
    tensor aligned to 256 bytes; write a step's values into ``host[name]``
    and call ``upload()``; the library calls take ``dev[name]``.  ``out`` is
    a pinned host tensor for the step's result (``download(out_dev)``)."""

    ORDER = ("q", "k_new", "v_new", "slot_mapping", "context_lens", "block_tables")

    def __init__(self, specs: dict, out_shape, out_dtype, device="cuda"):
        # specs: name -> (shape, dtype)
        offs, off = {}, 0
        for name in self.ORDER:
            shape, dtype = specs[name]
            n = 1
            for d in shape:
                n *= int(d)
            nbytes = n * torch.empty((), dtype=dtype).element_size()
            offs[name] = (off, nbytes, shape, dtype)
            off += (nbytes + 255) // 256 * 256
        self.nbytes = off
        self.host_buf = torch.empty(off, dtype=torch.uint8).pin_memory()
        self.dev_buf = torch.empty(off, dtype=torch.uint8, device=device)
        self.host, self.dev = {}, {}
        for name, (o, nb, shape, dtype) in offs.items():
            self.host[name] = self.host_buf[o:o + nb].view(dtype).view(*shape)
            self.dev[name] = self.dev_buf[o:o + nb].view(dtype).view(*shape)
        self.out = torch.empty(out_shape, dtype=out_dtype).pin_memory()

    @property
    def upload_bytes(self) -> int:
        return self.nbytes

    def upload(self, stream=None):
        s = stream or torch.cuda.current_stream()
        with torch.cuda.stream(s):
            self.dev_buf.copy_(self.host_buf, non_blocking=True)

    def download(self, out_dev: torch.Tensor, stream=None):
        s = stream or torch.cuda.current_stream()
        with torch.cuda.stream(s):
            self.out.copy_(out_dev, non_blocking=True)
