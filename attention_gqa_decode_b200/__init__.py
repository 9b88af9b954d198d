"""B200 (sm_100a) grouped-query attention: prefill and decode through a C ABI.

The work happens in ``libgqa_b200.so`` (hand-written CUDA for sm_100a, see
``include/gqa.h``).  This package is a thin ctypes binding with the same
names: it checks dtypes, devices and shapes, passes device pointers and the
current CUDA stream, and raises on any non-zero status.  PyTorch is used only
for device memory and streams.  There is no CPU fallback: if the library is
missing, importing the binding's entry points fails loudly.
"""
from ._lib import (GQAError, decode, decode_fp8, decode_paged, decode_split, gqa_decode,  # noqa: F401
                   gqa_decode_fp8, gqa_decode_fp8_rows, gqa_decode_split, gqa_decode_split_workspace_bytes, gqa_decode_paged, gqa_decode_paged_fp8, gqa_decode_rows,
                   gqa_get_device_status, gqa_mla_decode, gqa_mla_decode_path, gqa_mla_decode_rows, gqa_mla_decode_split,
                   gqa_mla_decode_split_workspace_bytes, gqa_prefill,
                   gqa_prefill_paged,
                   gqa_status_string, lib, library_path, load_library, mla_decode, prefill, prefill_paged)

__all__ = ["prefill", "prefill_paged", "decode", "decode_split", "decode_fp8", "decode_paged", "mla_decode",
           "gqa_prefill", "gqa_decode_split", "gqa_decode_split_workspace_bytes",
           "gqa_prefill_paged", "gqa_mla_decode", "gqa_mla_decode_rows", "gqa_mla_decode_path",
           "gqa_mla_decode_split", "gqa_mla_decode_split_workspace_bytes",
           "gqa_decode", "gqa_decode_rows", "gqa_decode_fp8", "gqa_decode_fp8_rows",
           "gqa_decode_paged", "gqa_decode_paged_fp8", "gqa_status_string", "gqa_get_device_status",
           "GQAError", "lib", "library_path", "load_library"]
