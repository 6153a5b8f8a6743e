"""Plain CPU fp64 oracle for paged MLA decode — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
(``cpu_baseline`` and ``--impl reference``) may import this package.  The product
path (``paged_kv_mla_create_b200``) never imports it and shares no code with it:
the arithmetic lives in ``mla_oracle.c`` (plain C, fp64, OpenMP over rows), and
this module only marshals numpy arrays into it.

Every function here follows the SGLang FlashMLA attention backend page
(flashmla_backend.py): the page table of ``init_forward_metadata``, the
``get_mla_metadata`` scheduler outputs, and ``flash_mla_with_kvcache`` as called
from ``forward_decode`` / ``forward_extend``; the partial-state merge follows the
``merge_state`` identity of the FlashInfer backend page (flashinfer_backend.py,
``forward_extend``).  Pins (tests/test_oracle_pins.py) tie each function to facts
fixed by the pages and by mathematics, not to this code.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

# The fixed per-piece overhead of the split planner, in 64-token blocks (the stated
# reading of get_mla_metadata's cost model; the CUDA planner defines its own copy).
FIXED_OVERHEAD_BLOCKS = 5
PAGE_SIZE = 64


def build(force: bool = False) -> str:
    """Compile mla_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", _LIB_PATH,
               _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    # A planted-mistake test points this at a deliberately broken copy of the oracle
    # to check that the pins catch it.
    override = os.environ.get("MLA_ORACLE_LIB_OVERRIDE")
    lib = ctypes.CDLL(override if override else build())
    P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
    lib.oracle_build_block_table.argtypes = [P, I64, P, P, I64, I64, P, I64, I64, I64]
    lib.oracle_build_block_table.restype = None
    lib.oracle_num_sm_parts.argtypes = [I64, I64, I64]
    lib.oracle_num_sm_parts.restype = I64
    lib.oracle_get_mla_metadata.argtypes = [P, I64, I64, I64, P, P]
    lib.oracle_get_mla_metadata.restype = None
    lib.oracle_mla_decode_rows.argtypes = [P, I32, P, I32, D, D, P, I64, P, P, P, P, I64, I64, I64,
                                           I64, I64, D, I32, I64, P, P, P]
    lib.oracle_mla_decode_rows.restype = I32
    lib.oracle_merge_states.argtypes = [I64, I64, P, P, P, P]
    lib.oracle_merge_states.restype = None
    lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_to_double.restype = D
    lib.oracle_e5m2_to_double.argtypes = [ctypes.c_uint8]
    lib.oracle_e5m2_to_double.restype = D
    lib.oracle_quantize_fp8.argtypes = [D, I32]
    lib.oracle_quantize_fp8.restype = ctypes.c_uint8
    lib.oracle_set_kv_buffer.argtypes = [P, I32, I64, I64, P, I64, P, I64, I32, ctypes.c_float]
    lib.oracle_set_kv_buffer.restype = None
    lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_double.restype = D
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = I32
    _lib = lib
    return lib


def _np(x, dtype):
    """Contiguous numpy array of the given dtype from a numpy array or CPU torch tensor."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if str(x.dtype) in ("torch.bfloat16", "torch.float8_e4m3fn", "torch.float8_e5m2"):
            import torch
            x = x.view(torch.uint16 if x.dtype == torch.bfloat16 else torch.uint8)
        x = x.numpy()
    return np.ascontiguousarray(x, dtype=dtype)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use."""
    return int(_load().oracle_num_threads())


def e4m3_to_double(code: int) -> float:
    return _load().oracle_e4m3_to_double(code)


def bf16_to_double(bits: int) -> float:
    return _load().oracle_bf16_to_double(bits)


def e5m2_to_double(code: int) -> float:
    return _load().oracle_e5m2_to_double(code)


FP8_FORMATS = {"e4m3": 1, "e5m2": 2}


def quantize_fp8(x: float, fmt: str = "e4m3") -> int:
    """The code of x rounded to the 8-bit format (nearest, ties to even, saturating)."""
    return int(_load().oracle_quantize_fp8(float(x), FP8_FORMATS[fmt]))


def _kv_format(kv_cache, kv_is_fp8):
    dt = str(getattr(kv_cache, "dtype", ""))
    if dt == "torch.float8_e5m2":
        return 2
    return 1 if kv_is_fp8 else 0


def set_kv_buffer(pool, cache_loc, k, k_scale=None):
    """Write the new tokens' rows k [n, dim] (bf16) at pool rows cache_loc [n]; pool is a
    torch tensor [slots, dim] of bf16, float8_e4m3fn or float8_e5m2 (modified in place,
    CPU).  An fp8 pool stores k / k_scale rounded to its format."""
    import torch
    fmt = {torch.bfloat16: 0, torch.float8_e4m3fn: 1, torch.float8_e5m2: 2}[pool.dtype]
    raw = pool.view(torch.uint16 if fmt == 0 else torch.uint8)
    assert raw.is_contiguous()
    arr = raw.numpy()   # shares memory with pool
    loc = _np(cache_loc, np.int64).reshape(-1)
    kb = _np(k, np.uint16)
    dim = arr.shape[-1]
    _load().oracle_set_kv_buffer(_ptr(arr), fmt, arr.size // dim, dim, _ptr(loc), loc.shape[0], _ptr(kb),
                                 kb.shape[-1], int(k_scale is not None),
                                 float(k_scale) if k_scale is not None else 1.0)
    return pool


def build_block_table(req_to_token, req_pool_indices, seq_lens, max_pages: int,
                      seq_len_add: int = 0, page_size: int = PAGE_SIZE) -> np.ndarray:
    """int32 [bs, max_pages] page table, -1 beyond each request's pages."""
    r2t = _np(req_to_token, np.int32)
    rpi = _np(req_pool_indices, np.int64)
    sl = _np(seq_lens, np.int64)
    bs = rpi.shape[0]
    out = np.empty((bs, max_pages), dtype=np.int32)
    _load().oracle_build_block_table(_ptr(r2t), r2t.shape[1], _ptr(rpi), _ptr(sl), seq_len_add,
                                     bs, _ptr(out), max_pages, max_pages, page_size)
    return out


def num_sm_parts(sm_count: int, num_heads_per_head_k: int, num_heads_k: int = 1) -> int:
    return int(_load().oracle_num_sm_parts(sm_count, num_heads_per_head_k, num_heads_k))


def get_mla_metadata(cache_seqlens, num_parts: int,
                     fixed_overhead: int = FIXED_OVERHEAD_BLOCKS):
    """(tile_scheduler_metadata int32 [num_parts, 8], num_splits int32 [bs+1])."""
    sl = _np(cache_seqlens, np.int32)
    bs = sl.shape[0]
    md = np.zeros((num_parts, 8), dtype=np.int32)
    ns = np.zeros((bs + 1,), dtype=np.int32)
    _load().oracle_get_mla_metadata(_ptr(sl), bs, num_parts, fixed_overhead, _ptr(md), _ptr(ns))
    return md, ns


def mla_decode_rows(q, kv_cache, req_to_token, req_pool_indices, cache_seqlens, row_ids,
                    softmax_scale: float, causal: bool, head_dim_v: int = 512,
                    kv_is_fp8: bool = False, descale_q: float = 1.0, descale_k: float = 1.0,
                    key_begin=None, key_end=None, q_is_fp8: bool = False):
    """Attention for the flat rows (b * q_len + i) * h + head of q [bs, q_len, h, dq].

    kv_cache is the token-slot pool (any shape whose last dim is dq; bf16, e4m3 or e5m2
    torch tensors, or the raw uint16 / uint8 bits of bf16 / e4m3 ones); q is bf16, or e4m3 codes with
    q_is_fp8 (descale_q then being the scale q was quantised with).  Returns
    (o [n, dv] fp64, lse [n] fp64).
    """
    qb = _np(q, np.uint8 if q_is_fp8 else np.uint16)
    bs, q_len, h, dq = qb.shape
    kv_format = _kv_format(kv_cache, kv_is_fp8)
    kv = _np(kv_cache, np.uint8 if kv_format else np.uint16).reshape(-1, dq)
    r2t = _np(req_to_token, np.int32)
    rpi = _np(req_pool_indices, np.int64)
    sl = _np(cache_seqlens, np.int32)
    rows = _np(row_ids, np.int64).reshape(-1)
    kb = _np(key_begin, np.int64) if key_begin is not None else None
    ke = _np(key_end, np.int64) if key_end is not None else None
    n = rows.shape[0]
    o = np.empty((n, head_dim_v), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = _load().oracle_mla_decode_rows(
        _ptr(qb), int(q_is_fp8), _ptr(kv), kv_format, float(descale_q), float(descale_k), _ptr(r2t),
        r2t.shape[1], _ptr(rpi), _ptr(sl), _ptr(kb) if kb is not None else None,
        _ptr(ke) if ke is not None else None, bs, q_len, h, dq, head_dim_v, float(softmax_scale),
        int(causal), n, _ptr(rows), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle: unsupported head_dim")
    return o, lse


def mla_decode(q, kv_cache, req_to_token, req_pool_indices, cache_seqlens, softmax_scale: float,
               causal: bool, head_dim_v: int = 512, kv_is_fp8: bool = False,
               descale_q: float = 1.0, descale_k: float = 1.0, key_begin=None, key_end=None,
               q_is_fp8: bool = False):
    """All rows: (o [bs, q_len, h, dv] fp64, lse [bs, q_len, h] fp64)."""
    bs, q_len, h, _ = tuple(q.shape)
    rows = np.arange(bs * q_len * h, dtype=np.int64)
    o, lse = mla_decode_rows(q, kv_cache, req_to_token, req_pool_indices, cache_seqlens, rows,
                             softmax_scale, causal, head_dim_v, kv_is_fp8, descale_q, descale_k,
                             key_begin, key_end, q_is_fp8)
    return o.reshape(bs, q_len, h, head_dim_v), lse.reshape(bs, q_len, h)


def merge_states(o_parts, lse_parts):
    """Merge n partial states of one row: o_parts [n, dv], lse_parts [n] -> (o [dv], lse)."""
    op = _np(o_parts, np.float64)
    lp = _np(lse_parts, np.float64).reshape(-1)
    n, dv = op.shape
    o = np.empty((dv,), dtype=np.float64)
    lse = np.empty((1,), dtype=np.float64)
    _load().oracle_merge_states(n, dv, _ptr(op), _ptr(lp), _ptr(o), _ptr(lse))
    return o, float(lse[0])
