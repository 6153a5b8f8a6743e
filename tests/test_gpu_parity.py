"""Parity of the CUDA path (through the C ABI) with the CPU fp64 oracle.

Page table and split plan: bit-exact.  Attention: max-abs 2e-2 and relative-L2 5e-3 on
o and on lse (fp8 caches, and e4m3 queries, are compared with the oracle run on the same
e4m3 codes and descales, i.e. on the dequantised values).  Small cases are compared element by element;
the five full-size workloads, in the launch configuration the benchmark times, are
compared on sampled rows that the oracle computes one by one."""
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_mla_create_b200 import workloads as W

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3
# Extend merges two bf16 partial results (each part's o is rounded to bf16, as the page's
# merge_state receives them, then the merged o again): two roundings of outputs that stay
# below 8 in magnitude are up to 2 x 2^-6 apart from one rounding, so the element bound doubles.
EXTEND_MAX_ABS = 4e-2


@pytest.fixture(scope="module")
def mla():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import paged_kv_mla_create_b200 as m
    m.library()
    return m


def run_path(mla, wl, parts=None):
    """The hot path exactly as the benchmark runs it: page table, plan, attention."""
    g = wl.to("cuda")
    bt = mla.build_block_table(g.req_to_token, g.req_pool_indices, g.seq_lens, wl.max_pages,
                               seq_len_add=wl.num_draft_tokens)
    md, ns = mla.get_mla_metadata(g.cache_seqlens, wl.q_len * wl.h, 1, wl.is_fp8,
                                  num_parts=parts)
    o, lse = mla.mla_decode_paged(g.q, g.kv_cache, bt, g.cache_seqlens, 512, md, ns,
                                  wl.softmax_scale, wl.causal, g.descale_q, g.descale_k)
    torch.cuda.synchronize()
    return bt.cpu().numpy(), md.cpu().numpy(), ns.cpu().numpy(), o.float().cpu().numpy(), \
        lse.cpu().numpy()


def oracle_rows(wl, rows):
    return oracle.mla_decode_rows(
        wl.q, wl.kv_cache, wl.req_to_token, wl.req_pool_indices, wl.cache_seqlens, rows,
        wl.softmax_scale, wl.causal, kv_is_fp8=wl.is_fp8,
        descale_q=float(wl.descale_q[0]) if wl.descale_q is not None else 1.0,
        descale_k=float(wl.descale_k[0]) if wl.descale_k is not None else 1.0,
        q_is_fp8=wl.q_is_fp8)


def assert_close(o_gpu, lse_gpu, o_ref, lse_ref, what="", max_abs=MAX_ABS):
    o_gpu = o_gpu.reshape(o_ref.shape)
    lse_gpu = lse_gpu.reshape(lse_ref.shape)
    dead = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), dead), f"{what}: -inf lse pattern differs"
    assert np.all(o_gpu[dead] == 0), f"{what}: rows without keys must be zero"
    live = ~dead
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite output"
    err = np.abs(o_gpu - o_ref)
    assert err.max() <= max_abs, f"{what}: o max-abs {err.max():.3e}"
    rel = np.linalg.norm(o_gpu - o_ref) / max(np.linalg.norm(o_ref), 1e-30)
    assert rel <= REL_L2, f"{what}: o rel-L2 {rel:.3e}"
    if live.any():
        lerr = np.abs(lse_gpu[live] - lse_ref[live])
        assert lerr.max() <= max_abs, f"{what}: lse max-abs {lerr.max():.3e}"
        lrel = np.linalg.norm(lse_gpu[live] - lse_ref[live]) / max(np.linalg.norm(lse_ref[live]), 1e-30)
        assert lrel <= REL_L2, f"{what}: lse rel-L2 {lrel:.3e}"


def check_metadata(mla, wl, bt, md, ns, parts=None):
    ref_bt = oracle.build_block_table(wl.req_to_token, wl.req_pool_indices, wl.seq_lens,
                                      wl.max_pages, seq_len_add=wl.num_draft_tokens)
    assert np.array_equal(bt, ref_bt), "page table differs from the oracle"
    P = parts if parts is not None else oracle.num_sm_parts(mla.sm_count(), wl.q_len * wl.h, 1)
    ref_md, ref_ns = oracle.get_mla_metadata(wl.cache_seqlens, P)
    assert np.array_equal(md, ref_md), "scheduler metadata differs from the oracle"
    assert np.array_equal(ns, ref_ns), "num_splits differs from the oracle"


def check_full(mla, wl, parts=None):
    bt, md, ns, o, lse = run_path(mla, wl, parts)
    check_metadata(mla, wl, bt, md, ns, parts)
    ref_o, ref_lse = oracle.mla_decode(wl.q, wl.kv_cache, wl.req_to_token, wl.req_pool_indices,
                                       wl.cache_seqlens, wl.softmax_scale, wl.causal,
                                       kv_is_fp8=wl.is_fp8,
                                       descale_q=float(wl.descale_q[0]) if wl.descale_q is not None else 1.0,
                                       descale_k=float(wl.descale_k[0]) if wl.descale_k is not None else 1.0,
                                       q_is_fp8=wl.q_is_fp8)
    assert_close(o, lse, ref_o, ref_lse, wl.name)
    assert mla.read_device_error() == 0


# ------------------------------------------------------------------ small, element by element
def test_tiny_workload(mla):
    check_full(mla, W.make_workload(1))


def test_tiny_workload_poisoned(mla):
    check_full(mla, W.make_workload(1, poison=True))


@pytest.mark.parametrize("lens", [[1], [63], [64], [65], [1, 63, 64, 65, 127, 128, 129],
                                  [300, 5, 1000, 64 * 9 + 1]])
def test_ragged_lengths(mla, lens):
    check_full(mla, W.make_case(lens, h=128, seed=21, poison=True))


@pytest.mark.parametrize("h", [16, 64, 128])
def test_head_counts(mla, h):
    check_full(mla, W.make_case([700, 65, 1300], h=h, seed=22, poison=True))


@pytest.mark.parametrize("parts", [1, 2, 3, 7, 74])
def test_forced_splits(mla, parts):
    """Few parts put many requests in one part; many parts split every request."""
    check_full(mla, W.make_case([2000, 33, 700, 4000, 129], h=128, seed=23, poison=True), parts)


def test_more_parts_than_sms_and_a_request_of_many_pieces(mla):
    """200 parts (400 CTAs, in waves: more than the SMs hold at once) split a 40000-token request
    into 157 pieces. That is more than the merge kernel keeps in registers, so the lse values past
    the first 128 pieces are reloaded and merged in further rounds."""
    wl = W.make_case([40000, 3000], h=16, seed=31)
    ref_md, ref_ns = oracle.get_mla_metadata(wl.cache_seqlens.numpy(), 200)
    assert int(ref_ns[1] - ref_ns[0]) > 128
    check_full(mla, wl, 200)


@pytest.mark.parametrize("q_len,h", [(4, 128), (2, 128), (3, 16), (4, 40)])
def test_target_verify(mla, q_len, h):
    check_full(mla, W.make_case([1000, 62, 129, 1], h=h, q_len=q_len, verify=True, seed=24,
                                poison=True))


def test_non_causal_multi_query(mla):
    wl = W.make_case([500, 70], h=32, q_len=3, verify=True, seed=25)
    wl.causal = False
    check_full(mla, wl)


@pytest.mark.parametrize("lens,h,q_len", [([37, 130], 16, 1), ([1, 63, 64, 65, 127, 128, 129], 128, 1),
                                         ([2000, 33, 700, 4000, 129], 128, 1), ([1000, 62, 129, 1], 128, 4)])
def test_fp8_cache(mla, lens, h, q_len):
    """e4m3 cache with a per-tensor scale; compared with the oracle on the same codes."""
    check_full(mla, W.make_case(lens, h=h, q_len=q_len, kv="fp8", verify=q_len > 1, seed=31,
                                poison=True))


@pytest.mark.parametrize("lens,h,q_len", [([37, 130], 16, 1), ([1, 63, 64, 65, 127, 128, 129], 128, 1),
                                         ([1000, 62, 129, 1], 128, 4), ([300, 5000], 40, 3)])
def test_fp8_queries(mla, lens, h, q_len):
    """e4m3 queries against an e4m3 cache (the backend page's fp8 branch: q quantised with the
    cache's scale): S on e4m3 x e4m3 tensor cores; the oracle runs on the same codes."""
    check_full(mla, W.make_case(lens, h=h, q_len=q_len, kv="fp8", verify=q_len > 1, seed=51,
                                poison=True, q_fp8=True))


@pytest.mark.parametrize("parts", [2, 7, 74])
def test_fp8_queries_forced_splits(mla, parts):
    check_full(mla, W.make_case([2000, 33, 700, 4000, 129], h=128, kv="fp8", seed=52, poison=True,
                                q_fp8=True), parts)


def test_fp8_cache_forced_splits(mla):
    check_full(mla, W.make_case([2000, 33, 700, 4000, 129], h=128, kv="fp8", seed=32, poison=True), 7)


def test_zero_length_request(mla):
    check_full(mla, W.make_case([0, 100, 0, 64], h=128, seed=26))


def test_large_scores_rescale(mla):
    wl = W.make_case([3000, 900], h=128, seed=27)
    wl.q.mul_(6.0)  # pushes running maxima up repeatedly: exercises the O rescale
    check_full(mla, wl)


def test_idle_batch(mla):
    wl = W.make_case([], h=128, seed=28)
    g = wl.to("cuda")
    bt = mla.build_block_table(g.req_to_token, g.req_pool_indices, g.seq_lens, 1)
    md, ns = mla.get_mla_metadata(g.cache_seqlens, 128)
    o, lse = mla.mla_decode_paged(g.q, torch.zeros(64, 576, dtype=torch.bfloat16, device="cuda"),
                                  bt, g.cache_seqlens, 512, md, ns, wl.softmax_scale, True)
    torch.cuda.synchronize()
    assert o.shape == (0, 1, 128, 512) and ns.cpu().tolist() == [0]


def test_bad_page_id_is_reported_not_faulted(mla):
    """A page id outside the pool (made on the host) must neither fault nor read
    outside the pool: the tile reads as zeros and the error word records it."""
    wl = W.make_case([130], h=128, seed=29)
    g = wl.to("cuda")
    bt = mla.build_block_table(g.req_to_token, g.req_pool_indices, g.seq_lens, wl.max_pages)
    bt[0, 1] = wl.kv_cache.shape[0] + 5
    md, ns = mla.get_mla_metadata(g.cache_seqlens, 128)
    o, lse = mla.mla_decode_paged(g.q, g.kv_cache, bt, g.cache_seqlens, 512, md, ns,
                                  wl.softmax_scale, True)
    torch.cuda.synchronize()
    assert mla.read_device_error() & 1
    assert torch.isfinite(o.float()).all()
    assert mla.read_device_error() == 0   # the word clears on read


@pytest.mark.parametrize("lens,h,q_len", [([37, 130], 16, 1), ([1, 63, 64, 65, 127, 128, 129], 128, 1),
                                         ([1000, 62, 129, 1], 128, 4)])
def test_e5m2_cache(mla, lens, h, q_len):
    """An e5m2 cache (the other fp8 type the backend accepts) with its per-tensor scale."""
    check_full(mla, W.make_case(lens, h=h, q_len=q_len, kv="e5m2", verify=q_len > 1, seed=53, poison=True))


def test_e5m2_cache_forced_splits(mla):
    check_full(mla, W.make_case([2000, 33, 700, 4000, 129], h=128, kv="e5m2", seed=54, poison=True), 7)


# ------------------------------------------------------------------ KV-cache write
def _raw(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.uint8)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float8_e4m3fn, torch.float8_e5m2])
@pytest.mark.parametrize("loc_dtype", [torch.int32, torch.int64])
def test_set_kv_buffer_bit_exact(mla, dtype, loc_dtype):
    """set_kv_buffer writes exactly the oracle's rows (fp8: k / k_scale rounded in float32 to
    the nearest code, ties to even, saturating) and nothing else."""
    rng = np.random.default_rng(60)
    slots, n = 64 * 40, 37
    pool = torch.from_numpy(rng.standard_normal((slots, 576)).astype(np.float32)).to(dtype)
    loc = torch.from_numpy(rng.choice(slots, size=n, replace=False)).to(loc_dtype)
    k = torch.from_numpy((rng.standard_normal((n, 576)) * 3).astype(np.float32)).to(torch.bfloat16)
    k[0, :8] = torch.tensor([1e30, -1e30, 0.0, -0.0, 1e-30, 448.0, 449.0, 57344.0]).to(torch.bfloat16)
    scale = torch.tensor([0.0123], dtype=torch.float32) if dtype != torch.bfloat16 else None
    ref = oracle.set_kv_buffer(pool.clone(), loc, k, float(scale[0]) if scale is not None else None)
    got = mla.set_kv_buffer(pool.cuda(), loc.cuda(), k.cuda(), scale.cuda() if scale is not None else None)
    torch.cuda.synchronize()
    assert torch.equal(_raw(got.cpu()), _raw(ref))
    assert mla.read_device_error() == 0


def test_set_kv_buffer_out_of_range_slot_is_reported(mla):
    pool = torch.zeros((128, 576), dtype=torch.bfloat16, device="cuda")
    k = torch.ones((3, 576), dtype=torch.bfloat16, device="cuda")
    loc = torch.tensor([5, 128, -1], dtype=torch.int64, device="cuda")
    mla.set_kv_buffer(pool, loc, k)
    torch.cuda.synchronize()
    assert mla.read_device_error() == 256
    assert torch.all(pool[5] == 1) and int(torch.count_nonzero(pool)) == 576


@pytest.mark.parametrize("kv", ["bf16", "fp8", "e5m2"])
def test_kv_write_then_attention(mla, kv):
    """One decode step as the backend runs it: each request's newest token (position L - 1) is
    written into the pool by set_kv_buffer, then attention reads it as the last key; the
    oracle does the same on its own copy of the pool."""
    wl = W.make_case([500, 64, 1300, 2], h=128, kv=kv, seed=61)
    rng = np.random.default_rng(61)
    k_new = torch.from_numpy(rng.standard_normal((wl.bs, 576)).astype(np.float32)).to(torch.bfloat16)
    slots = torch.tensor([int(wl.req_to_token[wl.req_pool_indices[b], int(wl.cache_seqlens[b]) - 1])
                          for b in range(wl.bs)], dtype=torch.int64)
    scale = wl.descale_k
    ref_pool = oracle.set_kv_buffer(wl.kv_cache.clone().reshape(-1, 576), slots, k_new,
                                    float(scale[0]) if scale is not None else None)
    g = wl.to("cuda")
    mla.set_kv_buffer(g.kv_cache.reshape(-1, 576), slots.cuda(), k_new.cuda(), g.descale_k)
    wl.kv_cache = ref_pool.reshape(wl.kv_cache.shape)
    bt = mla.build_block_table(g.req_to_token, g.req_pool_indices, g.seq_lens, wl.max_pages)
    md, ns = mla.get_mla_metadata(g.cache_seqlens, wl.q_len * wl.h, 1, wl.is_fp8)
    o, lse = mla.mla_decode_paged(g.q, g.kv_cache, bt, g.cache_seqlens, 512, md, ns, wl.softmax_scale,
                                  True, g.descale_q, g.descale_k)
    torch.cuda.synchronize()
    assert torch.equal(_raw(g.kv_cache.cpu()), _raw(wl.kv_cache))
    ref_o, ref_lse = oracle.mla_decode(wl.q, wl.kv_cache, wl.req_to_token, wl.req_pool_indices,
                                       wl.cache_seqlens, wl.softmax_scale, True, kv_is_fp8=wl.is_fp8,
                                       descale_q=float(wl.descale_q[0]) if wl.descale_q is not None else 1.0,
                                       descale_k=float(wl.descale_k[0]) if wl.descale_k is not None else 1.0)
    assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_lse, f"write then attend ({kv})")
    assert mla.read_device_error() == 0


# ------------------------------------------------------------------ full-size workloads
def sample_rows(wl, n, seed):
    """n random rows, plus, for every request and every query position, its first head, its
    last head and one random head: every request, every draft position and both ends of the
    head range are compared with the oracle."""
    rng = np.random.default_rng(seed)
    total = wl.bs * wl.q_len * wl.h
    rows = [rng.choice(total, size=min(n, total), replace=False)]
    for b in range(wl.bs):
        for i in range(wl.q_len):
            base = (b * wl.q_len + i) * wl.h
            rows.append(np.array([base, base + wl.h - 1, base + int(rng.integers(0, wl.h))]))
    return np.unique(np.concatenate(rows)).astype(np.int64)


@pytest.mark.parametrize("index", [2, 3, 4, 5])
def test_full_size_workload_sampled(mla, index):
    wl = W.make_workload(index)
    bt, md, ns, o, lse = run_path(mla, wl)
    check_metadata(mla, wl, bt, md, ns)
    rows = sample_rows(wl, 96 if index != 3 else 40, seed=index)
    ref_o, ref_lse = oracle_rows(wl, rows)
    o_rows = o.reshape(-1, 512)[rows]
    lse_rows = lse.reshape(-1)[rows]
    assert_close(o_rows, lse_rows, ref_o, ref_lse, wl.name)
    # properties that hold at any size: finite outputs everywhere, lse at least the
    # log of one allowed key's weight (lse > -inf) for every live row
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    assert mla.read_device_error() == 0


def test_full_size_fp8_queries_sampled(mla):
    """The fp8-cache workload with its queries handed over as e4m3 codes."""
    wl = W.make_workload(4, q_fp8=True)
    bt, md, ns, o, lse = run_path(mla, wl)
    check_metadata(mla, wl, bt, md, ns)
    rows = sample_rows(wl, 96, seed=44)
    ref_o, ref_lse = oracle_rows(wl, rows)
    assert_close(o.reshape(-1, 512)[rows], lse.reshape(-1)[rows], ref_o, ref_lse, wl.name)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    assert mla.read_device_error() == 0


# ------------------------------------------------------------------ degenerate and graph-mode cases
@pytest.mark.parametrize("parts", [None, 7])
def test_verify_rows_without_allowed_keys(mla, parts):
    """Causal multi-query rows whose limit L - q_len + i + 1 is <= 0 (a cache shorter than the
    draft) see no key: o = 0 and lse = -inf, as the oracle pins; the others see a prefix."""
    wl = W.make_case([2, 1, 3, 0, 100, 5, 700], h=128, q_len=4, verify=False, seed=41, poison=True)
    assert wl.causal and wl.num_draft_tokens == 0
    check_full(mla, wl, parts)


def _plan_with_lone_last_block(q_len):
    """A single request of L = 64k + 2 keys and a part count whose plan makes the request's
    final piece its last block alone: that piece holds only keys past the causal limit of
    draft rows i < q_len - 2, so those rows' partial state there is empty (lse = -inf)."""
    for k in range(2, 60):
        L = 64 * k + 2
        for parts in range(2, 40):
            md, ns = oracle.get_mla_metadata(np.array([L], dtype=np.int32), parts)
            if ns[1] < 2:
                continue
            last = [r for r in md if r[0] == 0 and r[2] == 1 and r[1] == k]   # piece [k, k+1)
            if last:
                return L, parts
    raise AssertionError("no plan with a one-block final piece")


def test_wholly_masked_split_piece(mla):
    L, parts = _plan_with_lone_last_block(4)
    wl = W.make_case([L - 4], h=128, q_len=4, verify=True, seed=42, poison=True)
    assert int(wl.cache_seqlens[0]) == L
    md, ns = oracle.get_mla_metadata(wl.cache_seqlens, parts)
    assert ns[1] >= 2
    check_full(mla, wl, parts)


def test_graph_mode_page_table(mla):
    """The graph-capture branch: a [max_bs, stride] table pre-filled with 1, a request-pool
    of 4096 rows, and fill_tail off: entries below cdiv(L, 64) match the oracle bit for bit,
    every other entry (also the columns past max_pages) keeps its 1."""
    wl = W.make_case([700, 65, 1, 0, 2049], h=16, seed=43)
    rng = np.random.default_rng(43)
    big_rows = rng.choice(4096, size=wl.bs, replace=False)
    r2t = torch.zeros((4096, wl.req_to_token.shape[1]), dtype=torch.int32)
    r2t[big_rows] = wl.req_to_token[wl.req_pool_indices]
    rpi = torch.tensor(big_rows, dtype=torch.int64)
    stride = wl.max_pages + 9
    table = torch.ones((wl.bs + 3, stride), dtype=torch.int32, device="cuda")
    out = table[:wl.bs, :wl.max_pages]
    mla.build_block_table(r2t.cuda(), rpi.cuda(), wl.seq_lens.cuda(), wl.max_pages, out=out,
                          fill_tail=False)
    torch.cuda.synchronize()
    got = table.cpu().numpy()
    ref = oracle.build_block_table(r2t, rpi, wl.seq_lens, wl.max_pages)
    npages = [-(-int(L) // 64) for L in wl.seq_lens]
    for b in range(wl.bs):
        assert np.array_equal(got[b, :npages[b]], ref[b, :npages[b]]), f"row {b}"
        assert np.all(got[b, npages[b]:] == 1), f"row {b}: tail overwritten"
    assert np.all(got[wl.bs:] == 1)
    assert mla.read_device_error() == 0


def test_misaligned_slots_are_reported(mla):
    """req_to_token whose slots for one page do not start a page: the entry is still
    slot / 64 (the oracle's value) and the error word records the broken precondition."""
    wl = W.make_case([300, 130], h=16, seed=44)
    r2t = wl.req_to_token.clone()
    row = int(wl.req_pool_indices[0])
    r2t[row, 64:128] += 1
    bt = mla.build_block_table(r2t.cuda(), wl.req_pool_indices.cuda(), wl.seq_lens.cuda(),
                               wl.max_pages)
    torch.cuda.synchronize()
    ref = oracle.build_block_table(r2t, wl.req_pool_indices, wl.seq_lens, wl.max_pages)
    assert np.array_equal(bt.cpu().numpy(), ref)
    assert mla.read_device_error() == 64
    assert mla.read_device_error() == 0


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_wait_that_runs_out_returns_with_an_error(mla, kv):
    """The failure path without a fault: a test hook makes every pair's leader withhold one
    page load, so a bounded wait (2 ms here) runs out; both CTAs of each pair stop, the kernel
    returns, the error word says MLA_DEVERR_WAIT_TIMEOUT, and the next ordinary call (with a
    zero-filled workspace) is correct again."""
    wl = W.make_case([2000, 1500, 900], h=128, kv=kv, seed=47)
    g = wl.to("cuda")
    bt = mla.build_block_table(g.req_to_token, g.req_pool_indices, g.seq_lens, wl.max_pages)
    md, ns = mla.get_mla_metadata(g.cache_seqlens, wl.q_len * wl.h, 1, wl.is_fp8, num_parts=2)
    try:
        mla.set_test_hooks(2_000_000, 3)
        mla.mla_decode_paged(g.q, g.kv_cache, bt, g.cache_seqlens, 512, md, ns, wl.softmax_scale, True,
                             g.descale_q, g.descale_k)
        torch.cuda.synchronize()
    finally:
        mla.set_test_hooks(0, -1)
    assert mla.read_device_error() & 16
    check_full(mla, wl, 2)


def test_q_out_of_f16_range_is_reported(mla):
    """With an e4m3 cache the product runs in f16: a q value beyond 65504 (made on the host)
    is recorded in the error word instead of silently overflowing."""
    wl = W.make_case([200, 70], h=16, kv="fp8", seed=45)
    wl.q[1, 0, 3, 17] = 70000.0
    run_path(mla, wl)
    assert mla.read_device_error() & 32


def test_fp8_cache_tiny_q_values(mla):
    """q values around 1e-6 (f16 subnormals in the e4m3 path) still meet the tolerance."""
    wl = W.make_case([300, 1000, 65], h=128, kv="fp8", seed=46)
    wl.q.mul_(1e-6)
    check_full(mla, wl)


# ------------------------------------------------------------------ planner, random batches
def test_planner_random_batches(mla):
    """The device split planner against the oracle's walk, bit-exact, on random batches:
    zero-length requests, single-block requests and long ones, 1 to 2500 requests (both the
    per-request walk and the part-by-part walk of batches above 2048), 1 to 148 parts."""
    rng = np.random.default_rng(20261202)
    for t in range(300):
        bs = int(rng.integers(1, 2500 if t % 25 == 0 else 300))
        kind = rng.integers(0, 4, size=bs)
        lens = np.where(kind == 0, 0, np.where(kind == 1, rng.integers(1, 65, size=bs),
                        np.where(kind == 2, rng.integers(1, 8193, size=bs), rng.integers(1, 131073, size=bs))))
        seqlens = torch.tensor(lens, dtype=torch.int32)
        parts = int(rng.integers(1, 149))
        md, ns = mla.get_mla_metadata(seqlens.cuda(), 128, num_parts=parts)
        ref_md, ref_ns = oracle.get_mla_metadata(seqlens.numpy(), parts)
        assert np.array_equal(md.cpu().numpy(), ref_md), f"batch {t}: metadata differs (bs {bs}, parts {parts})"
        assert np.array_equal(ns.cpu().numpy(), ref_ns), f"batch {t}: num_splits differs (bs {bs}, parts {parts})"


def test_planner_split_boundaries(mla):
    """The walk's split count by comparisons (a piece past a part's budget spans one or two
    further parts without a division, more with one): dense random batches whose requests are
    about 0, 1, 2 or 3 budgets long, give or take a few blocks, with the part count set so the
    budget lands near the one the lengths were drawn for.  Bit-exact against the oracle's
    part-by-part walk."""
    rng = np.random.default_rng(20261204)
    for t in range(3000):
        bs = int(rng.integers(1, 25))
        b0 = int(rng.integers(3, 201))
        nb = rng.integers(0, 4, size=bs) * b0 + rng.integers(-7, 8, size=bs)
        nb = np.maximum(nb, 0)
        lens = np.where(nb > 0, nb * 64 - rng.integers(0, 64, size=bs), 0)
        total = int(nb.sum()) + 5 * bs
        parts = int(min(148, max(1, round(total / b0) + int(rng.integers(-1, 2)))))
        seqlens = torch.tensor(lens, dtype=torch.int32)
        md, ns = mla.get_mla_metadata(seqlens.cuda(), 128, num_parts=parts)
        ref_md, ref_ns = oracle.get_mla_metadata(seqlens.numpy(), parts)
        assert np.array_equal(md.cpu().numpy(), ref_md), f"batch {t}: metadata differs (lens {lens.tolist()}, parts {parts})"
        assert np.array_equal(ns.cpu().numpy(), ref_ns), f"batch {t}: num_splits differs (lens {lens.tolist()}, parts {parts})"
    assert mla.read_device_error() == 0


# ------------------------------------------------------------------ one-launch metadata
@pytest.mark.parametrize("index", [1, 2, 3, 4, 5])
def test_one_launch_metadata_matches_oracle(mla, index):
    """build_decode_metadata: page table, int32 lengths and plan in one launch, bit-exact."""
    wl = W.make_workload(index)
    g = wl.to("cuda")
    bt, cl, md, ns = mla.build_decode_metadata(g.req_to_token, g.req_pool_indices, g.seq_lens,
                                               wl.max_pages, wl.q_len * wl.h, 1, wl.is_fp8,
                                               seq_len_add=wl.num_draft_tokens)
    torch.cuda.synchronize()
    check_metadata(mla, wl, bt.cpu().numpy(), md.cpu().numpy(), ns.cpu().numpy())
    assert np.array_equal(cl.cpu().numpy(), wl.cache_seqlens.numpy())
    assert mla.read_device_error() == 0


def _random_tables(rng, lens, extra_rows=3):
    """req_to_token / req_pool_indices for the given lengths: whole pages drawn from a
    shuffled pool, slots in order inside a page (no KV values: metadata only)."""
    pages = [-(-int(L) // 64) for L in lens]
    perm = rng.permutation(max(1, int(sum(pages) * 1.25) + 1))
    rows = len(lens) + extra_rows
    width = max(1, max(pages, default=1)) * 64
    r2t = np.zeros((rows, width), dtype=np.int32)
    rpi = rng.permutation(rows)[:len(lens)].astype(np.int64)
    cur = 0
    for b, n in enumerate(pages):
        pg = perm[cur:cur + n]
        cur += n
        if n:
            r2t[rpi[b], :64 * n] = (pg[:, None] * 64 + np.arange(64)[None, :]).reshape(-1)
    return torch.from_numpy(r2t), torch.from_numpy(rpi)


def test_one_launch_metadata_random_batches(mla):
    """The one-launch metadata against the oracle on random batches: zero, one-block and long
    requests, 1 to 2500 requests (both planner walks), 1 to 148 parts, a draft-token offset."""
    rng = np.random.default_rng(20261203)
    for t in range(60):
        bs = int(rng.integers(1, 2500 if t % 10 == 0 else 200))
        kind = rng.integers(0, 3, size=bs)
        lens = np.where(kind == 0, 0, np.where(kind == 1, rng.integers(1, 65, size=bs),
                                                rng.integers(1, 8193, size=bs)))
        add = int(rng.integers(0, 5)) if t % 3 == 0 else 0
        parts = int(rng.integers(1, 149))
        r2t, rpi = _random_tables(rng, lens + add)
        sl = torch.tensor(lens, dtype=torch.int32)
        max_pages = max(1, -(-int((lens + add).max()) // 64))
        bt, cl, md, ns = mla.build_decode_metadata(r2t.cuda(), rpi.cuda(), sl.cuda(), max_pages, 128,
                                                   seq_len_add=add, num_parts=parts)
        torch.cuda.synchronize()
        ref_bt = oracle.build_block_table(r2t, rpi, sl, max_pages, seq_len_add=add)
        ref_md, ref_ns = oracle.get_mla_metadata(lens + add, parts)
        assert np.array_equal(bt.cpu().numpy(), ref_bt), f"batch {t}: page table"
        assert np.array_equal(cl.cpu().numpy(), lens + add), f"batch {t}: lengths"
        assert np.array_equal(md.cpu().numpy(), ref_md), f"batch {t}: plan (bs {bs}, parts {parts})"
        assert np.array_equal(ns.cpu().numpy(), ref_ns), f"batch {t}: num_splits"
    assert mla.read_device_error() == 0


# ------------------------------------------------------------------ repeated calls, one workspace
def test_repeated_calls_on_one_workspace_are_identical(mla):
    """The path has no atomics and a fixed split order, so repeated calls must agree bit for
    bit; reusing one workspace also checks that a call never depends on what a previous call
    left in it (the merge drops the partials' L2 lines without writing them back)."""
    wl = W.make_case([700, 1500, 64, 2300, 1], 128, seed=77)
    g = wl.to("cuda")
    bt = mla.build_block_table(g.req_to_token, g.req_pool_indices, g.seq_lens, wl.max_pages)
    parts = 9   # forces several pieces per request
    md, ns = mla.get_mla_metadata(g.cache_seqlens, wl.q_len * wl.h, num_parts=parts)
    ws = torch.zeros((mla.workspace_bytes(wl.bs, wl.q_len, wl.h, parts),), dtype=torch.uint8, device="cuda")
    arrival = -(-wl.bs * 1 * 2 * 4 // 256) * 256   # leading arrival words [bs, query tiles, 2]
    outs = []
    for k in range(3):
        if k == 2:
            ws[arrival:].fill_(0xFF)   # partials full of NaN patterns must not matter either
        o, lse = mla.mla_decode_paged(g.q, g.kv_cache, bt, g.cache_seqlens, 512, md, ns, wl.softmax_scale,
                                      wl.causal, workspace=ws)
        torch.cuda.synchronize()
        outs.append((o.clone(), lse.clone()))
    for o, lse in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(lse, outs[0][1]), "repeated calls differ"
    assert int(ns[-1]) > wl.bs, "the case should split requests"
    assert torch.count_nonzero(ws[:arrival]) == 0, "every call leaves the arrival words zero"
    assert mla.read_device_error() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["decode", "verify", "fp8"])
def test_fold_in_and_stored_merge_agree_bit_for_bit(mla, case):
    """The last piece of a split request either folds the other pieces' partial rows into its own
    result or stores its partial and merges the stored ones at the end of its part; both sum the
    pieces in split-slot order with the same weights, so the results agree bit for bit (and
    whichever piece happens to finish last, the output is the same).  Nine forced parts give
    requests of two and three pieces (four in the verify case)."""
    if case == "decode":
        wl = W.make_case([700, 1500, 64, 2300, 1, 900], 128, seed=81)
    elif case == "verify":
        wl = W.make_case([700, 1500, 64, 2300, 3], 64, q_len=4, verify=True, seed=82)
    else:
        wl = W.make_case([700, 1500, 64, 2300, 1, 900], 128, kv="fp8", seed=83)
    g = wl.to("cuda")
    bt = mla.build_block_table(g.req_to_token, g.req_pool_indices, g.seq_lens, wl.max_pages,
                               seq_len_add=wl.num_draft_tokens)
    parts = 9
    md, ns = mla.get_mla_metadata(g.cache_seqlens, wl.q_len * wl.h, 1, wl.is_fp8, num_parts=parts)
    pieces = np.diff(ns.cpu().numpy())
    assert ({3, 4} if case == "verify" else {2, 3}) <= set(pieces.tolist()), pieces
    ws = torch.zeros((mla.workspace_bytes(wl.bs, wl.q_len, wl.h, parts),), dtype=torch.uint8, device="cuda")
    tiles = -(-(wl.q_len * wl.h) // 128)
    arrival = -(-wl.bs * tiles * 2 * 4 // 256) * 256
    outs = []
    try:
        for no_fold in (False, True, False):
            mla.set_test_hooks(0, -1, no_fold_in=no_fold)
            o, lse = mla.mla_decode_paged(g.q, g.kv_cache, bt, g.cache_seqlens, 512, md, ns, wl.softmax_scale,
                                          wl.causal, g.descale_q, g.descale_k, workspace=ws)
            torch.cuda.synchronize()
            assert torch.count_nonzero(ws[:arrival]) == 0, "every call leaves the arrival words zero"
            outs.append((o.clone(), lse.clone()))
    finally:
        mla.set_test_hooks(0, -1, no_fold_in=False)
    assert mla.read_device_error() == 0
    for o, lse in outs[1:]:
        assert torch.equal(o, outs[0][0]), "fold-in and stored merge differ"
        assert torch.equal(lse, outs[0][1]), "fold-in and stored merge differ (lse)"
    ref_o, ref_lse = oracle.mla_decode(wl.q, wl.kv_cache, wl.req_to_token, wl.req_pool_indices,
                                       wl.cache_seqlens, wl.softmax_scale, wl.causal, kv_is_fp8=wl.is_fp8,
                                       descale_q=float(wl.descale_q[0]) if wl.descale_q is not None else 1.0,
                                       descale_k=float(wl.descale_k[0]) if wl.descale_k is not None else 1.0)
    o, lse = outs[0]
    assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_lse, "fold-in " + case)


def test_random_split_batches(mla):
    """Random batches over forced part counts, so that requests split into one to many pieces in
    every arrangement the planner makes: each case against the oracle, then run again on the same
    workspace, which must give the same bits (whichever piece of a request happens to merge) and
    leave the arrival words zero."""
    rng = np.random.default_rng(2026)
    for case in range(24):
        h = int(rng.choice([16, 64, 128]))
        q_len = int(rng.choice([1, 1, 2]))
        bs = int(rng.integers(1, 7))
        lens = [int(x) for x in rng.choice([0, 1, 63, 64, 65, 200, 700, 1500, 2300], size=bs)]
        if max(lens) == 0:
            lens[0] = 129
        parts = int(rng.integers(2, 20))
        wl = W.make_case(lens, h, q_len=q_len, verify=q_len > 1, seed=3000 + case)
        g = wl.to("cuda")
        bt = mla.build_block_table(g.req_to_token, g.req_pool_indices, g.seq_lens, wl.max_pages,
                                   seq_len_add=wl.num_draft_tokens)
        md, ns = mla.get_mla_metadata(g.cache_seqlens, wl.q_len * wl.h, 1, False, num_parts=parts)
        ws = torch.zeros((mla.workspace_bytes(wl.bs, wl.q_len, wl.h, parts),), dtype=torch.uint8, device="cuda")
        tiles = -(-(wl.q_len * wl.h) // 128)
        arrival = -(-wl.bs * tiles * 2 * 4 // 256) * 256
        outs = []
        for _ in range(2):
            o, lse = mla.mla_decode_paged(g.q, g.kv_cache, bt, g.cache_seqlens, 512, md, ns, wl.softmax_scale,
                                          wl.causal, workspace=ws)
            torch.cuda.synchronize()
            assert torch.count_nonzero(ws[:arrival]) == 0, f"case {case}: arrival words left set"
            outs.append((o.clone(), lse.clone()))
        assert mla.read_device_error() == 0, f"case {case}"
        assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1]), f"case {case}: bits differ"
        ref_o, ref_lse = oracle.mla_decode(wl.q, wl.kv_cache, wl.req_to_token, wl.req_pool_indices,
                                           wl.cache_seqlens, wl.softmax_scale, wl.causal)
        assert_close(outs[0][0].float().cpu().numpy(), outs[0][1].cpu().numpy(), ref_o, ref_lse,
                     f"random case {case} (lens {lens}, h {h}, q_len {q_len}, parts {parts})")


def test_unzeroed_workspace_is_reported(mla):
    """A workspace whose arrival words are not zero (never zero-filled) is reported in the
    error word; zero-filling it makes the next call correct again."""
    wl = W.make_case([700, 1500, 64, 2300, 1], 128, seed=78)
    g = wl.to("cuda")
    bt = mla.build_block_table(g.req_to_token, g.req_pool_indices, g.seq_lens, wl.max_pages)
    parts = 9
    md, ns = mla.get_mla_metadata(g.cache_seqlens, wl.q_len * wl.h, num_parts=parts)
    ws = torch.full((mla.workspace_bytes(wl.bs, wl.q_len, wl.h, parts),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    mla.mla_decode_paged(g.q, g.kv_cache, bt, g.cache_seqlens, 512, md, ns, wl.softmax_scale,
                         wl.causal, workspace=ws)
    torch.cuda.synchronize()
    assert mla.read_device_error() & 128
    ws.zero_()
    o, lse = mla.mla_decode_paged(g.q, g.kv_cache, bt, g.cache_seqlens, 512, md, ns, wl.softmax_scale,
                                  wl.causal, workspace=ws)
    torch.cuda.synchronize()
    assert mla.read_device_error() == 0
    ref_o, ref_lse = oracle.mla_decode(wl.q, wl.kv_cache, wl.req_to_token, wl.req_pool_indices,
                                       wl.cache_seqlens, wl.softmax_scale, wl.causal)
    assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_lse, "after zero-fill")


# ------------------------------------------------------------------ extend (prefix + new rows) and merge_state
def test_merge_state_matches_oracle(mla):
    """merge_state of two partial results against the oracle's log-sum-exp merge (rows where
    one part, or both, saw no key included)."""
    rng = np.random.default_rng(81)
    rows = 300
    oa = torch.from_numpy(rng.standard_normal((rows, 512)).astype(np.float32)).to(torch.bfloat16)
    ob = torch.from_numpy(rng.standard_normal((rows, 512)).astype(np.float32)).to(torch.bfloat16)
    la = rng.normal(0.0, 3.0, rows).astype(np.float32)
    lb = rng.normal(0.0, 3.0, rows).astype(np.float32)
    la[::7] = -np.inf
    lb[::11] = -np.inf
    o, lse = mla.merge_state(oa.cuda(), torch.from_numpy(la).cuda(), ob.cuda(), torch.from_numpy(lb).cuda())
    torch.cuda.synchronize()
    ref_o = np.zeros((rows, 512))
    ref_lse = np.full((rows,), -np.inf)
    a64, b64 = oa.double().numpy(), ob.double().numpy()
    for r in range(rows):
        if np.isneginf(la[r]) and np.isneginf(lb[r]):
            continue
        ref_o[r], ref_lse[r] = oracle.merge_states(np.stack([a64[r], b64[r]]), np.array([la[r], lb[r]]))
    assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_lse, "merge_state")


def _new_rows(wl, prefix, e):
    """The new tokens' latent rows: the last e positions of each request in the combined cache."""
    pool = wl.kv_cache.reshape(-1, 576)
    slots = torch.tensor([[int(wl.req_to_token[wl.req_pool_indices[b], prefix[b] + i]) for i in range(e)]
                          for b in range(wl.bs)], dtype=torch.int64)
    return pool[slots.reshape(-1)].reshape(wl.bs, e, 576).contiguous()


@pytest.mark.parametrize("prefix,h,e", [([0, 130, 200, 64], 16, 37), ([300, 1, 0], 128, 64), ([513, 77], 40, 5),
                                        ([2048, 700], 128, 130)])
def test_extend_matches_attention_over_prefix_and_new_rows(mla, prefix, h, e):
    """Extend as the FlashInfer backend page writes it (ragged causal part over the new rows, paged
    part over the prefix, merge_state) against the oracle's single softmax over the prefix followed
    by the new rows, the new tokens causal: the target-verify form of the same cache."""
    wl = W.make_case(prefix, h=h, q_len=e, verify=True, seed=71 + e)
    k_new = _new_rows(wl, prefix, e)
    g = wl.to("cuda")
    mpp = max(1, max(-(-p // 64) for p in prefix))
    o, lse = mla.extend_paged_prefix(g.q, k_new.cuda(), g.kv_cache, g.req_to_token, g.req_pool_indices,
                                     torch.tensor(prefix, dtype=torch.int32).cuda(), mpp, wl.softmax_scale)
    torch.cuda.synchronize()
    ref_o, ref_lse = oracle.mla_decode(wl.q, wl.kv_cache, wl.req_to_token, wl.req_pool_indices, wl.cache_seqlens,
                                       wl.softmax_scale, True)
    assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_lse, f"extend {prefix} h={h} e={e}",
                 max_abs=EXTEND_MAX_ABS)
    assert mla.read_device_error() == 0


def test_extend_with_fp8_prefix(mla):
    """An e4m3 prefix with its descale and bf16 new rows: the oracle computes the two parts on
    their own (the ragged part over the new rows, causal; the paged part over the e4m3 prefix)
    and merges them with its log-sum-exp merge."""
    prefix, h, e = [150, 0, 64], 16, 9
    wl = W.make_case(prefix, h=h, q_len=e, verify=True, kv="fp8", seed=91)
    rng = np.random.default_rng(91)
    k_new = torch.from_numpy(rng.standard_normal((wl.bs, e, 576)).astype(np.float32)).to(torch.bfloat16)
    g = wl.to("cuda")
    mpp = max(1, max(-(-p // 64) for p in prefix))
    pl = torch.tensor(prefix, dtype=torch.int32)
    o, lse = mla.extend_paged_prefix(g.q, k_new.cuda(), g.kv_cache, g.req_to_token, g.req_pool_indices, pl.cuda(),
                                     mpp, wl.softmax_scale, descale_k=g.descale_k)
    torch.cuda.synchronize()
    dk = float(wl.descale_k[0])
    o2, l2 = oracle.mla_decode(wl.q, wl.kv_cache, wl.req_to_token, wl.req_pool_indices, pl.numpy(),
                               wl.softmax_scale, False, kv_is_fp8=True, descale_k=dk)
    r2t_new = np.arange(wl.bs * e, dtype=np.int32).reshape(wl.bs, e)
    o1, l1 = oracle.mla_decode(wl.q, k_new.reshape(-1, 576), r2t_new, np.arange(wl.bs), np.full(wl.bs, e, np.int32),
                               wl.softmax_scale, True)
    ref_o = np.zeros_like(o1)
    ref_lse = np.full(l1.shape, -np.inf)
    for idx in np.ndindex(l1.shape):
        if np.isneginf(l1[idx]) and np.isneginf(l2[idx]):
            continue
        ref_o[idx], ref_lse[idx] = oracle.merge_states(np.stack([o1[idx], o2[idx]]), np.array([l1[idx], l2[idx]]))
    assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_lse, "extend, e4m3 prefix",
                 max_abs=EXTEND_MAX_ABS)
    assert mla.read_device_error() == 0


# ------------------------------------------------------------------ one CUDA graph per step
def test_metadata_and_attention_in_one_graph_follow_new_batches(mla):
    """Metadata and attention captured in one CUDA graph, the way the benchmark replays a step:
    the attention kernel is a programmatic dependent of the metadata kernel, scheduled while the
    plan is still being computed.  Between replays the batch changes (new lengths, requests
    mapped to other rows of req_to_token), so an attention grid that read any of the plan, page
    table or lengths before the metadata grid had finished would attend the previous batch.
    Every replay is checked against the oracle for its own batch; the metadata bit for bit."""
    rng = np.random.default_rng(4242)
    lens = [3000, 700, 4100, 64, 1500, 2500, 130, 3900]
    wl = W.make_case(lens, 128, seed=4242)
    g = wl.to("cuda")
    alloc = {int(wl.req_pool_indices[b]): lens[b] for b in range(wl.bs)}
    batches = [(wl.req_pool_indices.clone(), wl.seq_lens.clone())]
    for _ in range(3):
        rpi = wl.req_pool_indices[torch.from_numpy(rng.permutation(wl.bs))]
        sl = torch.tensor([int(rng.integers(1, alloc[int(r)] + 1)) for r in rpi], dtype=torch.int32)
        batches.append((rpi.clone(), sl))
    batches.append(batches[0])
    rpi_d, sl_d = g.req_pool_indices.clone(), g.seq_lens.clone()
    parts = mla.num_sm_parts(wl.q_len * wl.h)
    bt = torch.empty((wl.bs, wl.max_pages), dtype=torch.int32, device="cuda")
    cl = torch.empty((wl.bs,), dtype=torch.int32, device="cuda")
    md = torch.empty((parts, 8), dtype=torch.int32, device="cuda")
    ns = torch.empty((wl.bs + 1,), dtype=torch.int32, device="cuda")
    o = torch.empty((wl.bs, 1, wl.h, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((wl.bs, 1, wl.h), dtype=torch.float32, device="cuda")
    ws = torch.zeros((mla.workspace_bytes(wl.bs, 1, wl.h, parts),), dtype=torch.uint8, device="cuda")

    def step():
        mla.build_decode_metadata(g.req_to_token, rpi_d, sl_d, wl.max_pages, wl.h, 1, False,
                                  out=(bt, cl, md, ns))
        mla.mla_decode_paged(g.q, g.kv_cache, bt, cl, 512, md, ns, wl.softmax_scale, True,
                             out=o, lse=lse, workspace=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    try:
        for t, (rpi, sl) in enumerate(batches):
            rpi_d.copy_(rpi)
            sl_d.copy_(sl)
            graph.replay()
            torch.cuda.synchronize()
            ref_bt = oracle.build_block_table(wl.req_to_token, rpi, sl, wl.max_pages)
            ref_md, ref_ns = oracle.get_mla_metadata(sl.numpy(), parts)
            assert np.array_equal(bt.cpu().numpy(), ref_bt), f"replay {t}: page table"
            assert np.array_equal(cl.cpu().numpy(), sl.numpy()), f"replay {t}: lengths"
            assert np.array_equal(md.cpu().numpy(), ref_md), f"replay {t}: plan"
            assert np.array_equal(ns.cpu().numpy(), ref_ns), f"replay {t}: num_splits"
            ref_o, ref_lse = oracle.mla_decode(wl.q, wl.kv_cache, wl.req_to_token, rpi, sl,
                                               wl.softmax_scale, True)
            assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_lse, f"replay {t}")
        assert int(ns[-1]) > 4 * wl.bs, "the batch should split requests into many pieces"
        assert mla.read_device_error() == 0
    finally:
        del graph
