"""Seeded synthetic decode and prefill workloads shared by the tests, the
benchmark and the oracle.  Input construction only; no attention arithmetic
lives here."""
from .workloads import (CONFIG_NAMES, DTYPE_BF16, DTYPE_F16, DTYPE_F32, PREFILL_NAMES, PagedDecodeCase,
                        PagedPrefillCase, algorithmic_bytes, bf16_bits_to_f32, build_case, build_prefill_case,
                        f32_to_bf16_bits, make_config, make_prefill_config, prefill_algorithmic)

__all__ = ["CONFIG_NAMES", "DTYPE_BF16", "DTYPE_F16", "DTYPE_F32", "PREFILL_NAMES", "PagedDecodeCase",
           "PagedPrefillCase", "algorithmic_bytes", "bf16_bits_to_f32", "build_case", "build_prefill_case",
           "f32_to_bf16_bits", "make_config", "make_prefill_config", "prefill_algorithmic"]
