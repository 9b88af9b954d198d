"""ctypes binding of libgqa_b200.so: argument marshalling only."""
from __future__ import annotations

import ctypes
import math
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libgqa_b200.so")
_lock = threading.Lock()
_handle = None

GQA_OK, GQA_ERR_INVALID_ARG, GQA_ERR_UNSUPPORTED, GQA_ERR_CUDA, GQA_ERR_TIMEOUT = range(5)

# every entry point include/gqa.h declares, with its ctypes signature
_vp, _i, _f, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int64, ctypes.c_size_t
SIGNATURES = {
    "gqa_prefill": ([_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp], _i),
    "gqa_decode": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp], _i),
    "gqa_decode_rows": ([_vp, _vp, _vp, _i64, _vp, _vp, _i, _i, _i, _i, _f, _vp], _i),
    "gqa_decode_split": ([_vp, _vp, _vp, _i64, _vp, _vp, _i, _i, _i, _i, _f, _vp, ctypes.c_size_t, _vp], _i),
    "gqa_decode_split_workspace_bytes": ([_i, _i, _i, _i], ctypes.c_size_t),
    "gqa_decode_split_noalloc": ([_vp, _vp, _vp, _i64, _vp, _vp, _i, _i, _i, _i, _f, _vp], _i),
    "gqa_decode_fp8": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp], _i),
    "gqa_decode_fp8_rows": ([_vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _vp], _i),
    "gqa_decode_paged": ([_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _i, _i, _i, _i, _f, _vp], _i),
    "gqa_decode_paged_fp8": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _i, _i, _i, _i, _f, _vp], _i),
    "gqa_prefill_paged": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp], _i),
    "gqa_mla_decode": ([_vp, _vp, _vp, _vp, _i, _i, _i, _f, _vp], _i),
    "gqa_mla_decode_rows": ([_vp, _vp, _i64, _vp, _vp, _i, _i, _i, _f, _vp], _i),
    "gqa_mla_decode_path": ([_i, _i, _i, _i64, _i], _i),
    "gqa_mla_decode_split": ([_vp, _vp, _i64, _vp, _vp, _i, _i, _i, _f, _vp, _sz, _vp], _i),
    "gqa_mla_decode_split_workspace_bytes": ([_i, _i, _i], _sz),
    "gqa_status_string": ([_i], ctypes.c_char_p),
    "gqa_get_device_status": ([_vp], _i),
}


class GQAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {gqa_status_string(status)} ({status})")


def library_path() -> str:
    return _LIB_PATH


def load_library(path: str) -> ctypes.CDLL:
    """A CDLL of a build of the library at `path` with every declared signature set."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m attention_gqa_decode_b200.build` (nvcc, sm_100a)")
    h = ctypes.CDLL(path)
    for name, (args, res) in SIGNATURES.items():
        fn = getattr(h, name)
        fn.argtypes = args
        fn.restype = res
    return h


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _handle
    with _lock:
        if _handle is None:
            _handle = load_library(_LIB_PATH)
    return _handle


def gqa_status_string(status: int) -> str:
    return lib().gqa_status_string(int(status)).decode()


def _stream_ptr(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def gqa_prefill(q, k, v, out, B, S_q, S_kv, h, n_kv, d_h, causal, scale, stream) -> int:
    """The raw C entry point (pointers as ints); returns the status code."""
    return lib().gqa_prefill(q, k, v, out, B, S_q, S_kv, h, n_kv, d_h, int(causal), float(scale), stream)


def gqa_decode(q, k_cache, v_cache, seqlens, out, B, h, n_kv, d_h, scale, stream) -> int:
    return lib().gqa_decode(q, k_cache, v_cache, seqlens, out, B, h, n_kv, d_h, float(scale), stream)


def gqa_decode_rows(q, k_cache, v_cache, cache_rows, seqlens, out, B, h, n_kv, d_h, scale, stream) -> int:
    return lib().gqa_decode_rows(q, k_cache, v_cache, int(cache_rows), seqlens, out, B, h, n_kv, d_h, float(scale),
                                 stream)


def gqa_decode_split(q, k_cache, v_cache, cache_rows, seqlens, out, B, h, n_kv, d_h, scale, workspace,
                     workspace_bytes, stream) -> int:
    return lib().gqa_decode_split(q, k_cache, v_cache, int(cache_rows), seqlens, out, B, h, n_kv, d_h, float(scale),
                                  workspace, int(workspace_bytes), stream)


def gqa_decode_split_workspace_bytes(B, h, n_kv, d_h) -> int:
    return int(lib().gqa_decode_split_workspace_bytes(B, h, n_kv, d_h))


def gqa_decode_fp8_rows(q, k_cache, v_cache, cache_rows, k_scale, v_scale, seqlens, out, B, h, n_kv, d_h, scale,
                        stream) -> int:
    return lib().gqa_decode_fp8_rows(q, k_cache, v_cache, int(cache_rows), k_scale, v_scale, seqlens, out, B, h, n_kv,
                                     d_h, float(scale), stream)


def gqa_mla_decode_rows(q_absorbed, c_kv, cache_rows, seqlens, out, B, h, d_c, scale, stream) -> int:
    return lib().gqa_mla_decode_rows(q_absorbed, c_kv, int(cache_rows), seqlens, out, B, h, d_c, float(scale), stream)


def gqa_mla_decode_path(B, h, d_c, cache_rows, with_workspace=0) -> int:
    return lib().gqa_mla_decode_path(B, h, d_c, int(cache_rows), int(with_workspace))


def gqa_mla_decode_split(q_absorbed, c_kv, cache_rows, seqlens, out, B, h, d_c, scale, workspace, workspace_bytes,
                         stream) -> int:
    return lib().gqa_mla_decode_split(q_absorbed, c_kv, int(cache_rows), seqlens, out, B, h, d_c, float(scale),
                                      workspace, workspace_bytes, stream)


def gqa_mla_decode_split_workspace_bytes(B, h, d_c) -> int:
    return lib().gqa_mla_decode_split_workspace_bytes(B, h, d_c)


def gqa_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, seqlens, out, B, h, n_kv, d_h, scale, stream) -> int:
    return lib().gqa_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, seqlens, out, B, h, n_kv, d_h,
                                float(scale), stream)


def gqa_decode_paged(q, k_pages, v_pages, block_table, max_blocks, page_size, num_pages, seqlens, out,
                     B, h, n_kv, d_h, scale, stream) -> int:
    return lib().gqa_decode_paged(q, k_pages, v_pages, block_table, max_blocks, page_size, num_pages, seqlens,
                                  out, B, h, n_kv, d_h, float(scale), stream)


def gqa_decode_paged_fp8(q, k_pages, v_pages, k_scale, v_scale, block_table, max_blocks, page_size, num_pages,
                         seqlens, out, B, h, n_kv, d_h, scale, stream) -> int:
    return lib().gqa_decode_paged_fp8(q, k_pages, v_pages, k_scale, v_scale, block_table, max_blocks, page_size,
                                      num_pages, seqlens, out, B, h, n_kv, d_h, float(scale), stream)


def gqa_prefill_paged(q, k_new, v_new, k_pages, v_pages, block_table, max_blocks, page_size, num_pages, past_lens,
                      out, B, S_q, h, n_kv, d_h, scale, stream) -> int:
    return lib().gqa_prefill_paged(q, k_new, v_new, k_pages, v_pages, block_table, max_blocks, page_size, num_pages,
                                   past_lens, out, B, S_q, h, n_kv, d_h, float(scale), stream)


def gqa_mla_decode(q_absorbed, c_kv, seqlens, out, B, h, d_c, scale, stream) -> int:
    return lib().gqa_mla_decode(q_absorbed, c_kv, seqlens, out, B, h, d_c, float(scale), stream)


def gqa_get_device_status(stream=None) -> int:
    return lib().gqa_get_device_status(_stream_ptr(stream))


def _check(t, name, ndim):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def prefill(q, k, v, causal: bool = True, scale: float | None = None, out=None, stream=None):
    """Exact attention for q [B,S_q,h,d], k/v [B,S_kv,n_kv,d] (bf16, CUDA); returns out [B,S_q,h,d].

    ``scale=None`` means 1/sqrt(d), the default of the flash_attn_func call
    shown on the toolsku page ("Flash Attention Usage", softmax_scale=None).
    """
    import torch
    _check(q, "q", 4), _check(k, "k", 4), _check(v, "v", 4)
    B, S_q, h, d = q.shape
    Bk, S_kv, n_kv, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk != d:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k, v must be on one device")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check(out, "out", 4)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    with torch.cuda.device(q.device):
        st = gqa_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, S_q, S_kv, h, n_kv, d,
                         causal, scale, _stream_ptr(stream))
    if st != GQA_OK:
        raise GQAError(st, "gqa_prefill")
    return out


# decode() sends a call to the split-KV kernels (gqa_decode_split) when the cache holds
# at least SPLIT_MIN_MEAN_ROWS rows per sequence and either the groups are mid-sized at
# d = 128 (SPLIT_WARP_GROUPS: the balanced warp-level kernel), wide (>= SPLIT_MIN_GROUP
# query heads per KV head) or there are too few (sequence, KV head) units for the
# cluster kernel's at most 8 splits each to reach every SM; everything else goes to the
# cluster kernel (gqa_decode_rows).  Measured on B200 (graph replay, caches rotated past
# L2): MQA B64 h32 L8192: split 4.60 TB/s, cluster 4.49; ragged B32 h64 n_kv1: split
# 2.15, cluster 1.27; B4 h64 n_kv1 L32768: split 2.07, cluster 0.39; G = 128: split 1.6,
# cluster 1.1; the GQA workload (G = 8): cluster 5.6, split 4.4.
SPLIT_WARP_GROUPS = (17, 64)
SPLIT_MIN_GROUP = 128
SPLIT_MIN_MEAN_ROWS = 256
_sm_counts = {}


def _sm_count(device) -> int:
    import torch
    dev = torch.device(device)
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    if key not in _sm_counts:
        _sm_counts[key] = torch.cuda.get_device_properties(key).multi_processor_count
    return _sm_counts[key]


def use_split(q, k_cache) -> bool:
    """The dispatch rule of decode() for q [B, h, d] and packed caches [T, n_kv, d]."""
    B, h, _ = q.shape
    T, n_kv, _ = k_cache.shape
    if n_kv <= 0 or h % n_kv or T < SPLIT_MIN_MEAN_ROWS * B:
        return False
    G = h // n_kv
    if q.shape[2] == 128 and SPLIT_WARP_GROUPS[0] <= G <= SPLIT_WARP_GROUPS[1]:
        return True
    units = B * n_kv * -(-G // 64)
    return G >= SPLIT_MIN_GROUP or units * 8 < _sm_count(q.device)


_workspaces = {}   # device index -> workspace tensor


def split_workspace(device, nbytes: int):
    """A device workspace of at least nbytes for gqa_decode_split: one per device, kept
    and grown as needed (it is scratch, so it needs no initialisation).  Calls that share
    it must not overlap on the GPU.  Make the first call of a shape before capturing a
    CUDA graph that uses it."""
    import torch
    dev = torch.device(device)
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=torch.device("cuda", key))
        _workspaces[key] = ws
    return ws


def decode_split(q, k_cache, v_cache, seqlens, scale: float | None = None, out=None, stream=None, workspace=None):
    """gqa_decode_split: the decode step with the batch's tokens divided evenly among
    the SMs (tensor-core products, partial results merged in a workspace).  Same
    arguments and result as :func:`decode`; ``workspace`` defaults to the binding's
    per-device workspace (:func:`split_workspace`)."""
    import torch
    _check(q, "q", 3), _check(k_cache, "k_cache", 3), _check(v_cache, "v_cache", 3)
    B, h, d = q.shape
    T, n_kv, dk = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape) or dk != d:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k_cache.shape)} v{tuple(v_cache.shape)}")
    _check_seqlens(seqlens, B)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check(out, "out", 3)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    with torch.cuda.device(q.device):
        need = gqa_decode_split_workspace_bytes(B, h, n_kv, d)
        ws = workspace if workspace is not None else split_workspace(q.device, need)
        st = gqa_decode_split(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), T, seqlens.data_ptr(),
                              out.data_ptr(), B, h, n_kv, d, scale, ws.data_ptr(), ws.numel() * ws.element_size(),
                              _stream_ptr(stream))
    if st != GQA_OK:
        raise GQAError(st, "gqa_decode_split")
    return out


def decode(q, k_cache, v_cache, seqlens, scale: float | None = None, out=None, stream=None):
    """One decode step: q [B,h,d], packed caches [T,n_kv,d], seqlens int32 [B] (CUDA).

    Returns out [B,h,d].  Sequence b's tokens start at cache row sum(seqlens[:b]);
    a sequence that would end past row T is cut there and GQA_ERR_INVALID_ARG is
    recorded in the device status word (gqa_get_device_status).  The call runs on
    gqa_decode_split or gqa_decode_rows by :func:`use_split` (the lengths stay on the
    device; the choice uses the shapes).
    """
    if q.dim() == 3 and k_cache.dim() == 3 and q.is_cuda and use_split(q, k_cache):
        return decode_split(q, k_cache, v_cache, seqlens, scale=scale, out=out, stream=stream)
    import torch
    _check(q, "q", 3), _check(k_cache, "k_cache", 3), _check(v_cache, "v_cache", 3)
    B, h, d = q.shape
    T, n_kv, dk = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape) or dk != d:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k_cache.shape)} v{tuple(v_cache.shape)}")
    if not isinstance(seqlens, torch.Tensor) or seqlens.dtype != torch.int32 or not seqlens.is_cuda \
            or seqlens.numel() != B or not seqlens.is_contiguous():
        raise ValueError("seqlens must be a contiguous int32 CUDA tensor with B entries")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check(out, "out", 3)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    with torch.cuda.device(q.device):
        st = gqa_decode_rows(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), T, seqlens.data_ptr(),
                             out.data_ptr(), B, h, n_kv, d, scale, _stream_ptr(stream))
    if st != GQA_OK:
        raise GQAError(st, "gqa_decode_rows")
    return out


def _check_cache(t, name, ndim, fp8):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    want = (torch.uint8, torch.float8_e4m3fn) if fp8 else (torch.bfloat16,)
    if t.dtype not in want:
        raise TypeError(f"{name} must be {' or '.join(map(str, want))}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_scales(k_scale, v_scale, n_kv):
    import torch
    for name, t in (("k_scale", k_scale), ("v_scale", v_scale)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or not t.is_cuda \
                or t.numel() != n_kv or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor with n_kv = {n_kv} entries")


def _check_seqlens(seqlens, B):
    import torch
    if not isinstance(seqlens, torch.Tensor) or seqlens.dtype != torch.int32 or not seqlens.is_cuda \
            or seqlens.numel() != B or not seqlens.is_contiguous():
        raise ValueError("seqlens must be a contiguous int32 CUDA tensor with B entries")


def decode_fp8(q, k_cache, v_cache, k_scale, v_scale, seqlens, scale: float | None = None, out=None,
               stream=None):
    """One decode step over packed E4M3 caches [sum(seqlens), n_kv, d] (uint8 codes or float8_e4m3fn).

    The value of a cached code of KV head g is code * k_scale[g] (K) or
    code * v_scale[g] (V); the scales are float32 [n_kv] CUDA tensors.  q is
    bf16 [B, h, d]; returns bf16 [B, h, d].
    """
    import torch
    _check_cache(k_cache, "k_cache", 3, True), _check_cache(v_cache, "v_cache", 3, True)
    _check(q, "q", 3)
    B, h, d = q.shape
    T, n_kv, dk = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape) or dk != d:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k_cache.shape)} v{tuple(v_cache.shape)}")
    _check_scales(k_scale, v_scale, n_kv)
    _check_seqlens(seqlens, B)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check(out, "out", 3)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    with torch.cuda.device(q.device):
        st = gqa_decode_fp8_rows(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), T, k_scale.data_ptr(),
                                 v_scale.data_ptr(), seqlens.data_ptr(), out.data_ptr(), B, h, n_kv, d, scale,
                                 _stream_ptr(stream))
    if st != GQA_OK:
        raise GQAError(st, "gqa_decode_fp8_rows")
    return out


def decode_paged(q, k_pages, v_pages, block_table, seqlens, scale: float | None = None, k_scale=None,
                 v_scale=None, out=None, stream=None):
    """One decode step over paged caches [num_pages, page_size, n_kv, d].

    Token t of sequence b is slot t % page_size of page block_table[b, t // page_size]
    (block_table: int32 [B, max_blocks] CUDA tensor).  bf16 pages, or E4M3
    pages (uint8 / float8_e4m3fn) with ``k_scale`` and ``v_scale`` float32 [n_kv].
    page_size must be a power of two in [16, 65536].  Returns bf16 [B, h, d].
    """
    import torch
    fp8 = k_pages.dtype in (torch.uint8, torch.float8_e4m3fn)
    _check(q, "q", 3)
    _check_cache(k_pages, "k_pages", 4, fp8), _check_cache(v_pages, "v_pages", 4, fp8)
    B, h, d = q.shape
    num_pages, page_size, n_kv, dk = k_pages.shape
    if tuple(v_pages.shape) != tuple(k_pages.shape) or dk != d:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k_pages.shape)} v{tuple(v_pages.shape)}")
    if not isinstance(block_table, torch.Tensor) or block_table.dtype != torch.int32 or not block_table.is_cuda \
            or block_table.dim() != 2 or block_table.shape[0] != B or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous int32 CUDA tensor [B, max_blocks]")
    _check_seqlens(seqlens, B)
    if fp8:
        _check_scales(k_scale, v_scale, n_kv)
    elif k_scale is not None or v_scale is not None:
        raise ValueError("scales apply to E4M3 pages only")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check(out, "out", 3)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    mb = block_table.shape[1]
    with torch.cuda.device(q.device):
        if fp8:
            st = gqa_decode_paged_fp8(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), k_scale.data_ptr(),
                                      v_scale.data_ptr(), block_table.data_ptr(), mb, page_size, num_pages,
                                      seqlens.data_ptr(), out.data_ptr(), B, h, n_kv, d, scale, _stream_ptr(stream))
        else:
            st = gqa_decode_paged(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), block_table.data_ptr(), mb,
                                  page_size, num_pages, seqlens.data_ptr(), out.data_ptr(), B, h, n_kv, d, scale,
                                  _stream_ptr(stream))
    if st != GQA_OK:
        raise GQAError(st, "gqa_decode_paged_fp8" if fp8 else "gqa_decode_paged")
    return out


def prefill_paged(q, k_new, v_new, k_pages, v_pages, block_table, past_lens, scale: float | None = None, out=None,
                  stream=None):
    """Chunked causal prefill over a paged bf16 cache, appending the chunk.

    q [B,S_q,h,d], k_new/v_new [B,S_q,n_kv,d], pages [num_pages,page_size,n_kv,d]
    (written in place at positions past_lens[b] .. past_lens[b]+S_q-1),
    block_table int32 [B,max_blocks], past_lens int32 [B] (CUDA).  Query row r
    attends to keys at positions <= past_lens[b] + r.  Returns out [B,S_q,h,d].
    """
    import torch
    _check(q, "q", 4), _check(k_new, "k_new", 4), _check(v_new, "v_new", 4)
    _check(k_pages, "k_pages", 4), _check(v_pages, "v_pages", 4)
    B, S_q, h, d = q.shape
    if tuple(k_new.shape) != tuple(v_new.shape) or k_new.shape[0] != B or k_new.shape[1] != S_q \
            or k_new.shape[3] != d:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k_new{tuple(k_new.shape)} v_new{tuple(v_new.shape)}")
    n_kv = k_new.shape[2]
    num_pages, page_size, n_kv_p, d_p = k_pages.shape
    if tuple(v_pages.shape) != tuple(k_pages.shape) or n_kv_p != n_kv or d_p != d:
        raise ValueError(f"page shape mismatch {tuple(k_pages.shape)} {tuple(v_pages.shape)}")
    if not isinstance(block_table, torch.Tensor) or block_table.dtype != torch.int32 or not block_table.is_cuda \
            or block_table.dim() != 2 or block_table.shape[0] != B or not block_table.is_contiguous():
        raise ValueError("block_table must be a contiguous int32 CUDA tensor [B, max_blocks]")
    _check_seqlens(past_lens, B)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check(out, "out", 4)
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    with torch.cuda.device(q.device):
        st = gqa_prefill_paged(q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), k_pages.data_ptr(),
                               v_pages.data_ptr(), block_table.data_ptr(), block_table.shape[1], page_size, num_pages,
                               past_lens.data_ptr(), out.data_ptr(), B, S_q, h, n_kv, d, scale, _stream_ptr(stream))
    if st != GQA_OK:
        raise GQAError(st, "gqa_prefill_paged")
    return out


def mla_decode(q_absorbed, c_kv, seqlens, scale: float | None = None, out=None, stream=None, workspace=None):
    """Absorbed MLA decode: q_absorbed [B,h,d_c], packed latent cache c_kv [sum(seqlens),d_c] (bf16,
    CUDA), seqlens int32 [B].  Returns softmax(q' c^T * scale) c as bf16 [B,h,d_c];
    ``scale=None`` is d_c ** -0.5.  Shapes for which gqa_mla_decode_path(..., 1) is 2
    run through gqa_mla_decode_split with ``workspace`` (default: the binding's
    per-device workspace, :func:`split_workspace`); the rest through gqa_mla_decode_rows."""
    import torch
    _check(q_absorbed, "q_absorbed", 3), _check(c_kv, "c_kv", 2)
    B, h, d_c = q_absorbed.shape
    if c_kv.shape[1] != d_c:
        raise ValueError(f"latent width mismatch q{tuple(q_absorbed.shape)} c_kv{tuple(c_kv.shape)}")
    _check_seqlens(seqlens, B)
    if scale is None:
        scale = float(d_c) ** -0.5
    if out is None:
        out = torch.empty_like(q_absorbed)
    else:
        _check(out, "out", 3)
        if out.shape != q_absorbed.shape:
            raise ValueError("out must have q_absorbed's shape")
    with torch.cuda.device(q_absorbed.device):
        if gqa_mla_decode_path(B, h, d_c, c_kv.shape[0], 1) == 2:
            need = gqa_mla_decode_split_workspace_bytes(B, h, d_c)
            ws = workspace if workspace is not None else split_workspace(q_absorbed.device, need)
            st = gqa_mla_decode_split(q_absorbed.data_ptr(), c_kv.data_ptr(), c_kv.shape[0], seqlens.data_ptr(),
                                      out.data_ptr(), B, h, d_c, scale, ws.data_ptr(), ws.numel() * ws.element_size(),
                                      _stream_ptr(stream))
            where = "gqa_mla_decode_split"
        else:
            st = gqa_mla_decode_rows(q_absorbed.data_ptr(), c_kv.data_ptr(), c_kv.shape[0], seqlens.data_ptr(),
                                     out.data_ptr(), B, h, d_c, scale, _stream_ptr(stream))
            where = "gqa_mla_decode_rows"
    if st != GQA_OK:
        raise GQAError(st, where)
    return out
