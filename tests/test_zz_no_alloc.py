"""The workspace-free attention entry point, for callers that cannot allocate device
memory when they run attention (engines that plan all device memory up front, plugin
hosts that forbid cudaMalloc in their execute hook).  It must give the same results as
the regular entry point, which takes a caller-allocated workspace, on two calls in a row
(the second call reuses the library's fixed scratch array as the first left it), and it
must refuse a problem too large for that array without launching anything.

This file is collected last on purpose, so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from paged_kv_mla_create_b200 import workloads as W

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3
NOALLOC_SCRATCH_BYTES = 64 << 20


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import paged_kv_mla_create_b200 as mla
    L = mla.library()
    P, I32, I64, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    L.mla_decode_paged_noalloc.argtypes = [P, I32, I32, I32, I32, I32, I32, P, I32, I64, I32, P,
                                           I64, I32, P, P, I32, P, F, I32, P, P, P, P, P]
    L.mla_decode_paged_noalloc.restype = I32
    return L


def _noalloc(lib, wl, g, bt, md, ns, out, lse):
    """One call of the workspace-free entry point straight through the C ABI."""
    p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    num_pages = g.kv_cache.numel() // (64 * 576)
    return lib.mla_decode_paged_noalloc(
        p(g.q), 0, wl.bs, wl.q_len, wl.h, 576, 512, p(g.kv_cache), 1 if wl.is_fp8 else 0,
        num_pages, 64, p(bt), bt.stride(0), bt.shape[1], p(g.cache_seqlens), p(md), md.shape[0],
        p(ns), wl.softmax_scale, int(wl.causal), p(g.descale_q), p(g.descale_k), p(out), p(lse),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(a, b):
    a = a.float().cpu().numpy()
    b = b.float().cpu().numpy()
    dead = np.isneginf(b)
    if dead.any():
        assert np.array_equal(np.isneginf(a), dead)
        a, b = a[~dead], b[~dead]
    assert np.abs(a - b).max() <= MAX_ABS
    assert np.linalg.norm(a - b) <= REL_L2 * max(np.linalg.norm(b), 1e-30)


@pytest.mark.parametrize("case", ["split_heavy", "dsv3_decode", "verify"])
def test_noalloc_matches_workspace_entry_point(lib, case):
    import paged_kv_mla_create_b200 as mla
    parts = None
    if case == "split_heavy":
        wl = W.make_case([2000, 33, 700, 4000, 129], h=128, seed=31, poison=True)
        parts = 7
    elif case == "dsv3_decode":
        wl = W.make_workload(2)
    else:
        wl = W.make_case([1000, 62, 129, 3000], h=128, q_len=4, verify=True, seed=32)
    g = wl.to("cuda")
    bt = mla.build_block_table(g.req_to_token, g.req_pool_indices, g.seq_lens, wl.max_pages,
                               seq_len_add=wl.num_draft_tokens)
    md, ns = mla.get_mla_metadata(g.cache_seqlens, wl.q_len * wl.h, 1, wl.is_fp8,
                                  num_parts=parts)
    assert mla.workspace_bytes(wl.bs, wl.q_len, wl.h, md.shape[0]) <= NOALLOC_SCRATCH_BYTES
    ref_o, ref_lse = mla.mla_decode_paged(g.q, g.kv_cache, bt, g.cache_seqlens, 512, md, ns,
                                          wl.softmax_scale, wl.causal, g.descale_q, g.descale_k)
    torch.cuda.synchronize()
    for call in range(2):
        out = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert _noalloc(lib, wl, g, bt, md, ns, out, lse) == 0, f"call {call}"
        torch.cuda.synchronize()
        _close(out, ref_o)
        _close(lse, ref_lse)
    assert mla.read_device_error() == 0


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    """4096 requests x 128 heads need ~1 GiB of split scratch: refused, nothing launched
    (the check comes before any pointer is touched)."""
    dummy = ctypes.c_void_p(256)
    status = lib.mla_decode_paged_noalloc(
        dummy, 0, 4096, 1, 128, 576, 512, dummy, 0, 1 << 16, 64, dummy, 64, 64, dummy, dummy, 74,
        dummy, 0.07, 1, None, None, dummy, dummy, None)
    assert status == 5  # MLA_ERR_WORKSPACE
