"""Paged MLA decode for B200 (sm_100a): page table, split-KV planner and attention.

A thin ctypes binding over the in-tree C-ABI library ``libmla_b200.so`` (declared in
``include/mla_b200.h``).  Every function here only marshals torch tensors into device
pointers and the current CUDA stream; all arithmetic runs in the library's kernels.
There is no CPU fallback: without the library, or without a CUDA device, the calls
raise.

The three entry points follow the calls of the SGLang FlashMLA attention backend page
(flashmla_backend.py):

* ``build_block_table``   — ``create_flashmla_kv_indices_triton`` in
  ``init_forward_metadata`` (block_kv_indices [bs, cdiv(max L, 64)], -1 padded);
* ``get_mla_metadata``    — ``get_mla_metadata(seq_lens, num_heads_per_head_k,
  num_heads_k, is_fp8_kvcache)`` returning (tile_scheduler_metadata, num_splits);
* ``mla_decode_paged``    — ``flash_mla_with_kvcache(q, k_cache, block_table,
  cache_seqlens, head_dim_v, tile_scheduler_metadata, num_splits, softmax_scale,
  causal, descale_q, descale_k)`` returning (o, lse); also exported under that name.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

from . import build as _build

__all__ = [
    "build_block_table", "get_mla_metadata", "build_decode_metadata", "mla_decode_paged",
    "flash_mla_with_kvcache", "set_kv_buffer",
    "num_sm_parts", "workspace_bytes", "read_device_error", "library", "MlaError",
]

PAGE_SIZE = 64
_STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_CUDA",
           4: "MLA_ERR_DEVICE_CHECK", 5: "MLA_ERR_WORKSPACE"}
DTYPE_BF16, DTYPE_FP8_E4M3, DTYPE_INT32, DTYPE_INT64, DTYPE_FP8_E5M2 = 0, 1, 2, 3, 4
_CACHE_DTYPES = {torch.bfloat16: DTYPE_BF16, torch.float8_e4m3fn: DTYPE_FP8_E4M3,
                 torch.float8_e5m2: DTYPE_FP8_E5M2}

_lib = None


class MlaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_STATUS.get(status, status)}")
        self.status = status


def library() -> ctypes.CDLL:
    """Load (building first when stale) the CUDA library; raises when it cannot."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB
    if _build.is_stale():
        path = _build.build()
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library missing: {path}")
    lib = ctypes.CDLL(path)
    P, I32, I64, F, SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                          ctypes.c_size_t)
    lib.mla_status_string.argtypes = [I32]
    lib.mla_status_string.restype = ctypes.c_char_p
    lib.mla_abi_version.argtypes = []
    lib.mla_abi_version.restype = I32
    lib.mla_build_block_table.argtypes = [P, I64, I64, P, I32, P, I32, I32, I32, P, I64, I32, I32,
                                          I32, P]
    lib.mla_build_block_table.restype = I32
    lib.mla_num_sm_parts.argtypes = [I32, I32, I32]
    lib.mla_num_sm_parts.restype = I32
    lib.mla_get_mla_metadata.argtypes = [P, I32, I32, I32, I32, I32, P, P, P]
    lib.mla_get_mla_metadata.restype = I32
    lib.mla_build_decode_metadata.argtypes = [P, I64, I64, P, I32, P, I32, I32, I32, P, I64, I32,
                                              I32, I32, I32, I32, I32, I32, P, P, P, P]
    lib.mla_build_decode_metadata.restype = I32
    lib.mla_decode_workspace_bytes.argtypes = [I32, I32, I32, I32]
    lib.mla_decode_workspace_bytes.restype = SZ
    lib.mla_decode_paged.argtypes = [P, I32, I32, I32, I32, I32, I32, P, I32, I64, I32, P, I64,
                                     I32, P, P, I32, P, F, I32, P, P, P, P, P, SZ, P]
    lib.mla_decode_paged.restype = I32
    lib.mla_set_kv_buffer.argtypes = [P, I32, I64, P, I32, I32, P, I64, P, P]
    lib.mla_set_kv_buffer.restype = I32
    lib.mla_merge_state.argtypes = [P, P, P, P, I64, I32, P, P, P]
    lib.mla_merge_state.restype = I32
    lib.mla_extend_workspace_bytes.argtypes = [I32, I32, I32, I32, I32]
    lib.mla_extend_workspace_bytes.restype = ctypes.c_size_t
    lib.mla_extend_paged_prefix.argtypes = [P, I32, I32, I32, P, P, I32, I64, P, I64, I64, P, I32, P, I32,
                                            ctypes.c_float, P, I32, P, P, P, ctypes.c_size_t, P]
    lib.mla_extend_paged_prefix.restype = I32
    lib.mla_set_test_hooks.argtypes = [ctypes.c_uint64, I32, I32]
    lib.mla_set_test_hooks.restype = I32
    lib.mla_read_device_error.argtypes = [ctypes.POINTER(I32), P]
    lib.mla_read_device_error.restype = I32
    _lib = lib
    return lib


def _check(status: int, what: str):
    if status != 0:
        raise MlaError(status, what)


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _require_cuda(*tensors):
    for t in tensors:
        if t is not None and not t.is_cuda:
            raise ValueError("paged_kv_mla_create_b200 runs on CUDA tensors only")


def _index_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.int32:
        return DTYPE_INT32
    if t.dtype == torch.int64:
        return DTYPE_INT64
    raise ValueError(f"index tensors must be int32 or int64, got {t.dtype}")


def sm_count(device=None) -> int:
    return torch.cuda.get_device_properties(device or torch.cuda.current_device()).multi_processor_count


def num_sm_parts(num_heads_per_head_k: int, num_heads_k: int = 1,
                 sm_count_: Optional[int] = None) -> int:
    """Rows of tile_scheduler_metadata for q_len * h_q = num_heads_per_head_k."""
    n = library().mla_num_sm_parts(sm_count_ if sm_count_ is not None else sm_count(),
                                   num_heads_per_head_k, num_heads_k)
    if n < 1:
        raise ValueError("invalid arguments to num_sm_parts")
    return n


def workspace_bytes(bs: int, q_len: int, h_q: int, parts: int) -> int:
    """Bytes of the attention workspace; allocate it zero-filled (torch.zeros) once, then
    reuse it: every completed call leaves its leading arrival words zero."""
    return int(library().mla_decode_workspace_bytes(bs, q_len, h_q, parts))


def build_block_table(req_to_token: torch.Tensor, req_pool_indices: torch.Tensor,
                      seq_lens: torch.Tensor, max_seqlen_pad: int, seq_len_add: int = 0,
                      out: Optional[torch.Tensor] = None, fill_tail: bool = True) -> torch.Tensor:
    """int32 [bs, max_seqlen_pad] page table: entry (b, p) is the page holding position 64p
    of request b (L_b = seq_lens[b] + seq_len_add); other entries are -1 when fill_tail."""
    _require_cuda(req_to_token, req_pool_indices, seq_lens, out)
    if req_to_token.dtype != torch.int32 or req_to_token.dim() != 2 or req_to_token.stride(1) != 1:
        raise ValueError("req_to_token must be a row-major int32 matrix")
    bs = int(req_pool_indices.shape[0])
    if out is None:
        out = torch.empty((bs, max_seqlen_pad), dtype=torch.int32, device=req_to_token.device)
    if out.dtype != torch.int32 or out.dim() != 2 or out.stride(1) != 1:
        raise ValueError("out must be a row-major int32 matrix")
    rpi = req_pool_indices.contiguous()
    sl = seq_lens.contiguous()
    _check(library().mla_build_block_table(
        _ptr(req_to_token), req_to_token.shape[0], req_to_token.stride(0), _ptr(rpi),
        _index_dtype(rpi), _ptr(sl), _index_dtype(sl), int(seq_len_add), bs, _ptr(out),
        out.stride(0), int(max_seqlen_pad), PAGE_SIZE, int(bool(fill_tail)),
        _stream(req_to_token.device)), "mla_build_block_table")
    return out


def get_mla_metadata(cache_seqlens: torch.Tensor, num_heads_per_head_k: int,
                     num_heads_k: int = 1, is_fp8_kvcache: bool = False,
                     num_parts: Optional[int] = None,
                     out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None):
    """(tile_scheduler_metadata int32 [num_sm_parts, 8], num_splits int32 [bs + 1]).

    The part count follows from the device's SM count; ``num_parts`` plans for that many
    parts instead (the SM count of a device with 2 SMs per part and query tile)."""
    _require_cuda(cache_seqlens)
    if cache_seqlens.dtype != torch.int32:
        raise ValueError("cache_seqlens must be int32 (the backend casts with .to(torch.int32))")
    if num_heads_per_head_k <= 0 or num_heads_k <= 0:
        raise ValueError("num_heads_per_head_k and num_heads_k must be positive")
    sl = cache_seqlens.contiguous()
    bs = int(sl.shape[0])
    dev = sl.device
    if num_parts is not None:
        m_tiles = -(-num_heads_per_head_k // 128)
        sms = 2 * m_tiles * num_heads_k * int(num_parts)
    else:
        sms = sm_count(dev)
    parts = num_sm_parts(num_heads_per_head_k, num_heads_k, sms)
    if out is None:
        md = torch.empty((parts, 8), dtype=torch.int32, device=dev)
        ns = torch.empty((bs + 1,), dtype=torch.int32, device=dev)
    else:
        md, ns = out
        if md.shape[0] != parts or ns.numel() != bs + 1:
            raise ValueError("out tensors do not match the plan's shapes")
    _check(library().mla_get_mla_metadata(_ptr(sl), bs, int(num_heads_per_head_k), int(num_heads_k),
                                          int(bool(is_fp8_kvcache)), sms, _ptr(md), _ptr(ns),
                                          _stream(dev)),
           "mla_get_mla_metadata")
    return md, ns


def build_decode_metadata(req_to_token: torch.Tensor, req_pool_indices: torch.Tensor,
                          seq_lens: torch.Tensor, max_seqlen_pad: int, num_heads_per_head_k: int,
                          num_heads_k: int = 1, is_fp8_kvcache: bool = False, seq_len_add: int = 0,
                          num_parts: Optional[int] = None, fill_tail: bool = True,
                          out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor]] = None):
    """The per-batch metadata in one launch: (block_table int32 [bs, max_seqlen_pad],
    cache_seqlens int32 [bs] = seq_lens + seq_len_add, tile_scheduler_metadata int32
    [num_sm_parts, 8], num_splits int32 [bs + 1]) -- what build_block_table, the int32 cast
    of the lengths and get_mla_metadata give."""
    _require_cuda(req_to_token, req_pool_indices, seq_lens)
    if req_to_token.dtype != torch.int32 or req_to_token.dim() != 2 or req_to_token.stride(1) != 1:
        raise ValueError("req_to_token must be a row-major int32 matrix")
    if num_heads_per_head_k <= 0 or num_heads_k <= 0:
        raise ValueError("num_heads_per_head_k and num_heads_k must be positive")
    dev = req_to_token.device
    bs = int(req_pool_indices.shape[0])
    if num_parts is not None:
        sms = 2 * (-(-num_heads_per_head_k // 128)) * num_heads_k * int(num_parts)
    else:
        sms = sm_count(dev)
    parts = num_sm_parts(num_heads_per_head_k, num_heads_k, sms)
    if out is None:
        bt = torch.empty((bs, max_seqlen_pad), dtype=torch.int32, device=dev)
        cl = torch.empty((bs,), dtype=torch.int32, device=dev)
        md = torch.empty((parts, 8), dtype=torch.int32, device=dev)
        ns = torch.empty((bs + 1,), dtype=torch.int32, device=dev)
    else:
        bt, cl, md, ns = out
    if bt.dtype != torch.int32 or bt.dim() != 2 or bt.stride(1) != 1:
        raise ValueError("block_table must be a row-major int32 matrix")
    if md.shape[0] != parts or ns.numel() != bs + 1 or (cl is not None and cl.numel() != bs):
        raise ValueError("out tensors do not match the metadata's shapes")
    rpi = req_pool_indices.contiguous()
    sl = seq_lens.contiguous()
    _check(library().mla_build_decode_metadata(
        _ptr(req_to_token), req_to_token.shape[0], req_to_token.stride(0), _ptr(rpi),
        _index_dtype(rpi), _ptr(sl), _index_dtype(sl), int(seq_len_add), bs, _ptr(bt), bt.stride(0),
        int(max_seqlen_pad), PAGE_SIZE, int(bool(fill_tail)), int(num_heads_per_head_k),
        int(num_heads_k), int(bool(is_fp8_kvcache)), sms, _ptr(cl), _ptr(md), _ptr(ns),
        _stream(dev)), "mla_build_decode_metadata")
    return bt, cl, md, ns


def mla_decode_paged(q: torch.Tensor, k_cache: torch.Tensor, block_table: torch.Tensor,
                     cache_seqlens: torch.Tensor, head_dim_v: int,
                     tile_scheduler_metadata: torch.Tensor, num_splits: torch.Tensor,
                     softmax_scale: float, causal: bool = True,
                     descale_q: Optional[torch.Tensor] = None,
                     descale_k: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None):
    """Paged MLA attention.  q bf16 [bs, q_len, h_q, 576], or float8_e4m3fn codes with an
    float8_e4m3fn cache (the backend's fp8 branch: q quantised with the cache's scale, that
    scale passed as descale_q and descale_k); k_cache bf16 or float8_e4m3fn with 576-wide
    token rows grouped in 64-token pages ([pages, 64, 576], [pages, 64, 1, 576] or
    [slots, 576]).  Returns (o bf16 [bs, q_len, h_q, 512], lse fp32 [bs, q_len, h_q])."""
    _require_cuda(q, k_cache, block_table, cache_seqlens, tile_scheduler_metadata, num_splits,
                  descale_q, descale_k, out, lse, workspace)
    if q.dim() != 4 or q.dtype not in (torch.bfloat16, torch.float8_e4m3fn) or not q.is_contiguous():
        raise ValueError("q must be a contiguous bf16 or float8_e4m3fn [bs, q_len, h_q, head_dim] tensor")
    bs, q_len, h_q, head_dim = (int(x) for x in q.shape)
    if not k_cache.is_contiguous() or k_cache.shape[-1] != head_dim:
        raise ValueError("k_cache must be contiguous with head_dim-wide rows")
    if k_cache.numel() % (PAGE_SIZE * head_dim):
        raise ValueError("k_cache must hold whole 64-token pages")
    num_pages = k_cache.numel() // (PAGE_SIZE * head_dim)
    if k_cache.dtype not in _CACHE_DTYPES:
        raise ValueError(f"unsupported k_cache dtype {k_cache.dtype}")
    kv_dtype = _CACHE_DTYPES[k_cache.dtype]
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.stride(1) != 1:
        raise ValueError("block_table must be a row-major int32 [bs, max_pages] matrix")
    if cache_seqlens.dtype != torch.int32:
        raise ValueError("cache_seqlens must be int32")
    for name, d in (("descale_q", descale_q), ("descale_k", descale_k)):
        if d is not None and (d.dtype != torch.float32 or d.numel() < 1):
            raise ValueError(f"{name} must be a float32 tensor of one element")
    dev = q.device
    parts = int(tile_scheduler_metadata.shape[0])
    if out is None:
        out = torch.empty((bs, q_len, h_q, head_dim_v), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((bs, q_len, h_q), dtype=torch.float32, device=dev)
    need = workspace_bytes(bs, q_len, h_q, parts) if bs else 0
    if workspace is None and need:
        # zero-filled: the leading arrival words must be zero at a workspace's first use
        workspace = torch.zeros((need,), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    sl = cache_seqlens.contiguous()
    q_dtype = DTYPE_FP8_E4M3 if q.dtype == torch.float8_e4m3fn else DTYPE_BF16
    _check(library().mla_decode_paged(
        _ptr(q), q_dtype, bs, q_len, h_q, head_dim, int(head_dim_v), _ptr(k_cache), kv_dtype,
        num_pages, PAGE_SIZE, _ptr(block_table), block_table.stride(0), int(block_table.shape[1]),
        _ptr(sl), _ptr(tile_scheduler_metadata), parts, _ptr(num_splits), float(softmax_scale),
        int(bool(causal)), _ptr(descale_q), _ptr(descale_k), _ptr(out), _ptr(lse),
        _ptr(workspace), ws_bytes, _stream(dev)), "mla_decode_paged")
    return out, lse


flash_mla_with_kvcache = mla_decode_paged


def set_kv_buffer(k_cache: torch.Tensor, cache_loc: torch.Tensor, k: torch.Tensor,
                  k_scale: Optional[torch.Tensor] = None) -> torch.Tensor:
    """token_to_kv_pool.set_kv_buffer for the MLA latent pool: row cache_loc[i] of k_cache
    ([slots, 576] or any view with 576-wide rows; bf16, float8_e4m3fn or float8_e5m2) receives
    k[i] (bf16 [n, 576], the latent row whose first 512 columns are the value), an fp8 pool
    storing k / k_scale rounded to its format.  In place; returns k_cache."""
    _require_cuda(k_cache, cache_loc, k, k_scale)
    if k_cache.dtype not in _CACHE_DTYPES or not k_cache.is_contiguous() or k_cache.shape[-1] != 576:
        raise ValueError("k_cache must be a contiguous bf16 / float8 pool with 576-wide rows")
    if k.dtype != torch.bfloat16 or k.dim() != 2 or k.shape[1] != 576 or k.stride(1) != 1:
        raise ValueError("k must be a bf16 [n, 576] matrix with unit column stride")
    if k_scale is not None and (k_scale.dtype != torch.float32 or k_scale.numel() < 1):
        raise ValueError("k_scale must be a float32 tensor of one element")
    loc = cache_loc.contiguous()
    n = int(k.shape[0])
    if loc.numel() != n:
        raise ValueError("one cache_loc entry per token")
    _check(library().mla_set_kv_buffer(_ptr(k_cache), _CACHE_DTYPES[k_cache.dtype], k_cache.numel() // 576,
                                       _ptr(loc), _index_dtype(loc), n, _ptr(k), k.stride(0), _ptr(k_scale),
                                       _stream(k_cache.device)), "mla_set_kv_buffer")
    return k_cache


def merge_state(o_a: torch.Tensor, lse_a: torch.Tensor, o_b: torch.Tensor, lse_b: torch.Tensor,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
    """merge_state(o1, s1, o2, s2) of two partial attention results of the same rows: bf16
    o [..., 512] and fp32 natural-log lse [...] (-inf: no key).  Returns (o, lse)."""
    _require_cuda(o_a, lse_a, o_b, lse_b, out, lse)
    for o_, l_ in ((o_a, lse_a), (o_b, lse_b)):
        if o_.dtype != torch.bfloat16 or not o_.is_contiguous() or o_.shape[-1] != 512:
            raise ValueError("o must be a contiguous bf16 [..., 512] tensor")
        if l_.dtype != torch.float32 or not l_.is_contiguous() or l_.numel() * 512 != o_.numel():
            raise ValueError("lse must be a contiguous float32 tensor of one value per row")
    if o_a.shape != o_b.shape:
        raise ValueError("the two parts must have the same shape")
    rows = lse_a.numel()
    if out is None:
        out = torch.empty_like(o_a)
    if lse is None:
        lse = torch.empty_like(lse_a)
    _check(library().mla_merge_state(_ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b), rows, 512, _ptr(out), _ptr(lse),
                                     _stream(o_a.device)), "mla_merge_state")
    return out, lse


def extend_workspace_bytes(bs: int, e: int, h_q: int, max_prefix_pages: int, sm_count_: Optional[int] = None) -> int:
    """Bytes of the extend workspace; allocate it zero-filled once and reuse it."""
    return int(library().mla_extend_workspace_bytes(bs, e, h_q, max_prefix_pages,
                                                    sm_count_ if sm_count_ is not None else sm_count()))


def extend_paged_prefix(q: torch.Tensor, k_new: torch.Tensor, k_cache: torch.Tensor, req_to_token: torch.Tensor,
                        req_pool_indices: torch.Tensor, prefix_lens: torch.Tensor, max_prefix_pages: int,
                        softmax_scale: float, descale_k: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None):
    """Extend with a cached prefix: q bf16 [bs, e, h_q, 576] of the e new tokens of every request
    attends the new tokens' latent rows k_new (bf16 [bs, e, 576]) causally and the request's
    prefix_lens[b] cached rows of k_cache (through req_to_token) in full; the two partial results
    are merged by merge_state.  Returns (o bf16 [bs, e, h_q, 512], lse fp32 [bs, e, h_q])."""
    _require_cuda(q, k_new, k_cache, req_to_token, req_pool_indices, prefix_lens, descale_k, out, lse, workspace)
    if q.dim() != 4 or q.dtype != torch.bfloat16 or not q.is_contiguous() or q.shape[-1] != 576:
        raise ValueError("q must be a contiguous bf16 [bs, e, h_q, 576] tensor")
    bs, e, h_q, _ = (int(x) for x in q.shape)
    if k_new.dtype != torch.bfloat16 or not k_new.is_contiguous() or tuple(k_new.shape) != (bs, e, 576):
        raise ValueError("k_new must be a contiguous bf16 [bs, e, 576] tensor")
    if k_cache.dtype not in _CACHE_DTYPES or not k_cache.is_contiguous() or k_cache.shape[-1] != 576:
        raise ValueError("k_cache must be a contiguous bf16 / float8 pool with 576-wide rows")
    if k_cache.numel() % (PAGE_SIZE * 576):
        raise ValueError("k_cache must hold whole 64-token pages")
    if req_to_token.dtype != torch.int32 or req_to_token.dim() != 2 or req_to_token.stride(1) != 1:
        raise ValueError("req_to_token must be a row-major int32 matrix")
    pl = prefix_lens.to(torch.int32).contiguous()
    rpi = req_pool_indices.contiguous()
    dev = q.device
    if out is None:
        out = torch.empty((bs, e, h_q, 512), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((bs, e, h_q), dtype=torch.float32, device=dev)
    need = extend_workspace_bytes(bs, e, h_q, int(max_prefix_pages)) if bs else 0
    if workspace is None and need:
        workspace = torch.zeros((need,), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(library().mla_extend_paged_prefix(
        _ptr(q), bs, e, h_q, _ptr(k_new), _ptr(k_cache), _CACHE_DTYPES[k_cache.dtype],
        k_cache.numel() // (PAGE_SIZE * 576), _ptr(req_to_token), int(req_to_token.shape[0]),
        req_to_token.stride(0), _ptr(rpi), _index_dtype(rpi), _ptr(pl), int(max_prefix_pages),
        float(softmax_scale), _ptr(descale_k), sm_count(dev), _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes,
        _stream(dev)), "mla_extend_paged_prefix")
    return out, lse


def set_test_hooks(wait_budget_ns: int = 0, withhold_tile: int = -1, no_fold_in: bool = False) -> None:
    """Test-only: the pipeline wait budget (0: the default 2 s), a tile whose page load the
    leader CTAs withhold (-1: none) and whether the last piece of a split request must merge by
    stored partials instead of folding the others in, for every later attention launch in this
    process."""
    _check(library().mla_set_test_hooks(int(wait_budget_ns), int(withhold_tile), int(bool(no_fold_in))),
           "mla_set_test_hooks")


def read_device_error(device=None) -> int:
    """Synchronise the current stream and return (and clear) the sticky device error word."""
    code = ctypes.c_int32(0)
    status = library().mla_read_device_error(ctypes.byref(code),
                                             _stream(device or torch.cuda.current_device()))
    if status not in (0, 4):
        raise MlaError(status, "mla_read_device_error")
    return int(code.value)
