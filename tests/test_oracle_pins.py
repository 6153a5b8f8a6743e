"""Pins for the CPU oracle: each test ties an oracle function to something other than
the oracle itself — library routines (torch's float8 / bf16 casts, scipy's softmax and
logsumexp), closed forms, invariants of attention, and worked examples under
tests/golden/.  CPU only."""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from paged_kv_mla_create_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- element decoding
def test_e4m3_decoding_matches_torch_for_all_codes():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_double(int(c)) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_bf16_decoding_matches_torch():
    rng = np.random.default_rng(0)
    bits = np.concatenate([np.arange(0, 65536, 97), rng.integers(0, 65536, 4000)]).astype(np.uint16)
    ref = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_e5m2_decoding_matches_torch_for_all_codes():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e5m2).to(torch.float64).numpy()
    got = np.array([oracle.e5m2_to_double(int(c)) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])   # infinities included


@pytest.mark.parametrize("fmt,tdt,top", [("e4m3", torch.float8_e4m3fn, 448.0),
                                          ("e5m2", torch.float8_e5m2, 57344.0)])
def test_fp8_rounding_matches_torch_and_saturates(fmt, tdt, top):
    """Round-to-nearest-even of in-range values agrees with torch's cast; exact midpoints
    between neighbouring codes go to the even code; beyond the range it saturates."""
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(3000) * top / 8, rng.standard_normal(3000) * 1e-3,
                        [0.0, -0.0, top, -top, 1e-12, -1e-12]])
    x = x[np.abs(x) <= top]
    ref = torch.from_numpy(x.astype(np.float32)).to(tdt).view(torch.uint8).numpy()
    got = np.array([oracle.quantize_fp8(float(np.float32(v)), fmt) for v in x], dtype=np.uint8)
    assert np.array_equal(got, ref)
    # midpoints: between every pair of neighbouring positive finite codes
    dec = oracle.e4m3_to_double if fmt == "e4m3" else oracle.e5m2_to_double
    vals = [dec(c) for c in range(0x80)]
    finite = [c for c in range(0x80) if math.isfinite(vals[c])]
    for a, b in zip(finite[:-1], finite[1:]):
        mid = (vals[a] + vals[b]) / 2
        want = a if a % 2 == 0 else b
        assert oracle.quantize_fp8(mid, fmt) == want, (fmt, a, b)
        assert oracle.quantize_fp8(-mid, fmt) == want | 0x80
    assert oracle.quantize_fp8(1e30, fmt) == finite[-1]
    assert oracle.quantize_fp8(-1e30, fmt) == finite[-1] | 0x80


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float8_e4m3fn, torch.float8_e5m2])
def test_set_kv_buffer_writes_the_new_rows(dtype):
    """Rows cache_loc[i] receive token i's row (k / k_scale rounded to an fp8 pool's format, as
    torch's cast rounds it); every other row, and out-of-range slots, are left alone."""
    rng = np.random.default_rng(11)
    slots, dim, n = 50, 576, 7
    pool = torch.from_numpy(rng.standard_normal((slots, dim)).astype(np.float32)).to(dtype)
    before = pool.clone()
    loc = np.array([3, 17, 0, 49, 8, 60, -2], dtype=np.int64)   # the last two are outside the pool
    k = torch.from_numpy(rng.standard_normal((n, dim)).astype(np.float32)).to(torch.bfloat16)
    scale = 0.0125 if dtype != torch.bfloat16 else None
    oracle.set_kv_buffer(pool, loc, k, scale)
    for i, s in enumerate(loc):
        if not 0 <= s < slots:
            continue
        if dtype == torch.bfloat16:
            want = k[i]
        else:
            want = (k[i].float() / torch.tensor(scale, dtype=torch.float32)).to(dtype)
        assert torch.equal(pool[s].view(torch.uint8 if dtype != torch.bfloat16 else torch.int16),
                           want.view(torch.uint8 if dtype != torch.bfloat16 else torch.int16)), (i, s)
    untouched = [s for s in range(slots) if s not in set(int(v) for v in loc)]
    assert torch.equal(pool[untouched].float(), before[untouched].float())


# ---------------------------------------------------------------- page table
def _parse_page_table_golden():
    lines = [l.split("#")[0].strip() for l in open(os.path.join(GOLDEN, "page_table_small.txt"))]
    lines = [l for l in lines if l]
    r2t = np.zeros((4, 192), dtype=np.int32)
    expect = {}
    for l in lines:
        key, rest = l.split(" ", 1)
        if key == "rows":
            for item in rest.split()[1:]:
                row, pages = item.split(":")
                for p_idx, page in enumerate(int(x) for x in pages.split(",")):
                    r2t[int(row), 64 * p_idx:64 * p_idx + 64] = 64 * page + np.arange(64)
        elif key == "rpi":
            rpi = np.array([int(x) for x in rest.split()], dtype=np.int64)
        elif key == "seq_lens":
            sl = np.array([int(x) for x in rest.split()], dtype=np.int64)
        else:
            expect[int(key[3:])] = np.array(
                [[int(x) for x in part.split()] for part in rest.split("|")], dtype=np.int32)
    return r2t, rpi, sl, expect


def test_page_table_golden():
    r2t, rpi, sl, expect = _parse_page_table_golden()
    for add, table in expect.items():
        got = oracle.build_block_table(r2t, rpi, sl, max_pages=table.shape[1], seq_len_add=add)
        assert np.array_equal(got, table), (add, got, table)


@pytest.mark.parametrize("lens", [[1, 63, 64, 65], [0, 5, 129], [300], [64 * 7]])
@pytest.mark.parametrize("add", [0, 4])
def test_page_table_reconstructs_slots(lens, add):
    """Every position j < L lies at slot 64 * bt[b, j // 64] + j % 64 (page-aligned pool),
    and every entry past the request's pages is -1."""
    wl = W.make_case([max(0, l) for l in lens], h=1, q_len=max(1, add), verify=add > 0, seed=3)
    L = wl.cache_seqlens.numpy().astype(np.int64)
    max_pages = int(max(1, -(-L.max() // 64)) + 2)
    bt = oracle.build_block_table(wl.req_to_token, wl.req_pool_indices, wl.seq_lens, max_pages,
                                  seq_len_add=add)
    r2t = wl.req_to_token.numpy()
    for b in range(len(lens)):
        npg = -(-L[b] // 64)
        assert np.all(bt[b, npg:] == -1)
        j = np.arange(L[b])
        assert np.array_equal(64 * bt[b, j // 64] + j % 64, r2t[wl.req_pool_indices[b], :L[b]])


# ---------------------------------------------------------------- planner
def _parse_planner_golden():
    rows, rest_row = {}, None
    for l in open(os.path.join(GOLDEN, "planner_tiny.txt")):
        l = l.split("#")[0].strip()
        if not l:
            continue
        k, *v = l.split()
        v = [int(x) for x in v]
        if k == "parts":
            parts, F = v
        elif k == "seqlens":
            sl = np.array(v, dtype=np.int32)
        elif k == "num_splits":
            ns = np.array(v, dtype=np.int32)
        elif k == "row":
            rows[v[0]] = v[1:]
        elif k == "rows_rest":
            rest_row = v
    md = np.array([rows.get(i, rest_row) for i in range(parts)], dtype=np.int32)
    return parts, F, sl, ns, md


def test_planner_golden_tiny():
    parts, F, sl, ns, md = _parse_planner_golden()
    assert oracle.num_sm_parts(148, 16, 1) == parts
    got_md, got_ns = oracle.get_mla_metadata(sl, parts, F)
    assert np.array_equal(got_ns, ns)
    assert np.array_equal(got_md, md)


def check_plan_invariants(sl, P, F, md, ns):
    """Exact cover of every request's blocks by the parts' pieces, in order, with no
    overlap; each part within its budget; num_splits counts the pieces."""
    bs = len(sl)
    blocks = [-(-max(int(L), 0) // 64) for L in sl]
    total = sum(b + F for b in blocks)
    payload = -(-total // P) + F
    pieces = [[] for _ in range(bs)]
    prev_end = (0, 0)
    for i in range(P):
        b0, k0, b1, k1, s0 = (int(x) for x in md[i, :5])
        assert (b0, k0) == prev_end, "parts must tile the request/block sequence in order"
        assert tuple(md[i, 5:]) == (0, 0, 0)
        cost = 0
        b, k, s = b0, k0, s0
        while (b, k) != (b1, k1):
            assert b < bs
            end = blocks[b] if b < b1 else k1
            assert end > k or blocks[b] == 0
            pieces[b].append((k, end, s))
            cost += end - k + F
            if b < b1:
                b, k, s = b + 1, 0, 0
            else:
                k = end
        assert cost <= payload
        prev_end = (b1, k1)
    assert prev_end == (bs, 0), "all requests must be covered within the parts"
    assert ns[0] == 0
    for b in range(bs):
        got = pieces[b]
        assert got[0][0] == 0 and got[-1][1] == blocks[b]
        for a, c in zip(got, got[1:]):
            assert a[1] == c[0]
        assert [p[2] for p in got] == list(range(len(got)))
        assert ns[b + 1] - ns[b] == len(got)
    assert ns[bs] <= bs + P - 1 or bs == 0


@pytest.mark.parametrize("seed", range(40))
def test_planner_invariants_random(seed):
    rng = np.random.default_rng(seed)
    bs = int(rng.integers(0, 70))
    kind = seed % 4
    if kind == 0:
        sl = rng.integers(1, 5000, bs)
    elif kind == 1:
        sl = rng.integers(1, 300, bs)
        if bs:
            sl[rng.integers(0, bs)] = int(rng.integers(50000, 200000))
    elif kind == 2:
        sl = rng.integers(0, 130, bs)
    else:
        sl = rng.choice([1, 63, 64, 65, 4096, 131072], bs)
    sl = sl.astype(np.int32)
    for P in (1, 2, 7, 18, 74, 148):
        for F in (0, 1, 5):
            md, ns = oracle.get_mla_metadata(sl, P, F)
            check_plan_invariants(sl, P, F, md, ns)


def test_planner_adversarial_overhead_chain():
    """A continuation piece that fits with less than F of budget left is the case in
    which a part can consume less than cdiv(total, P); coverage must still hold."""
    for bs in range(1, 12):
        for L0 in range(1, 40):
            sl = np.array([L0 * 64] + [64 * ((L0 * 7 + j) % 13 + 1) for j in range(bs - 1)],
                          dtype=np.int32)
            for P in (2, 3, 5, 8):
                md, ns = oracle.get_mla_metadata(sl, P, 5)
                check_plan_invariants(sl, P, 5, md, ns)


def test_num_sm_parts():
    assert oracle.num_sm_parts(148, 128, 1) == 74
    assert oracle.num_sm_parts(148, 512, 1) == 18
    assert oracle.num_sm_parts(148, 16, 1) == 74
    assert oracle.num_sm_parts(148, 129, 1) == 37


# ---------------------------------------------------------------- attention
def _decode_kv(wl):
    """Pool values in fp64 through torch's own casts (independent of the oracle)."""
    kv = wl.kv_cache.reshape(-1, 576).to(torch.float64)
    if wl.is_fp8:
        kv = kv * float(wl.descale_k[0])
    return kv.numpy()


def brute_force(wl, causal=True):
    """Attention via numpy gathers and scipy's softmax / logsumexp."""
    kv = _decode_kv(wl)
    q = wl.q.to(torch.float64).numpy()
    dq = float(wl.descale_q[0]) if wl.descale_q is not None else 1.0
    r2t = wl.req_to_token.numpy()
    bs, q_len, h, _ = q.shape
    o = np.zeros((bs, q_len, h, 512))
    lse = np.full((bs, q_len, h), -np.inf)
    for b in range(bs):
        L = int(wl.cache_seqlens[b])
        slots = r2t[int(wl.req_pool_indices[b]), :L]
        K = kv[slots]
        for i in range(q_len):
            lim = L - q_len + i + 1 if causal else L
            if lim <= 0:
                continue
            S = wl.softmax_scale * dq * (q[b, i] @ K[:lim].T)       # [h, lim]
            o[b, i] = scipy.special.softmax(S, axis=1) @ K[:lim, :512]
            lse[b, i] = scipy.special.logsumexp(S, axis=1)
    return o, lse


def run_oracle(wl, **kw):
    return oracle.mla_decode(
        wl.q, wl.kv_cache, wl.req_to_token, wl.req_pool_indices, wl.cache_seqlens,
        wl.softmax_scale, kw.pop("causal", True), kv_is_fp8=wl.is_fp8,
        descale_q=float(wl.descale_q[0]) if wl.descale_q is not None else 1.0,
        descale_k=float(wl.descale_k[0]) if wl.descale_k is not None else 1.0, **kw)


@pytest.mark.parametrize("case", [
    dict(lens=[37, 130], h=16),
    dict(lens=[1, 64, 65, 200], h=4),
    dict(lens=[70, 129], h=3, q_len=4, verify=True),
    dict(lens=[2, 100], h=2, q_len=3, verify=True),
    dict(lens=[90, 33], h=4, kv="fp8"),
])
def test_oracle_matches_scipy_brute_force(case):
    wl = W.make_case(case["lens"], case["h"], case.get("q_len", 1), case.get("kv", "bf16"),
                     case.get("verify", False), seed=11, poison=True)
    o, lse = run_oracle(wl)
    bo, blse = brute_force(wl)
    assert np.allclose(o, bo, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, blse, rtol=1e-12, atol=1e-12)


def test_tiny_workload_matches_brute_force():
    wl = W.make_workload(1)
    o, lse = run_oracle(wl)
    bo, blse = brute_force(wl)
    assert np.allclose(o, bo, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, blse, rtol=1e-12, atol=1e-12)


def test_seq_len_one_returns_first_token():
    wl = W.make_case([1, 1], h=8, seed=5)
    o, lse = run_oracle(wl)
    kv = _decode_kv(wl)
    q = wl.q.to(torch.float64).numpy()
    for b in range(2):
        slot = int(wl.req_to_token[int(wl.req_pool_indices[b]), 0])
        assert np.array_equal(o[b, 0], np.broadcast_to(kv[slot, :512], (8, 512)))
        expect = wl.softmax_scale * (q[b, 0] @ kv[slot])
        assert np.allclose(lse[b, 0], expect, rtol=0, atol=1e-12)


def test_equal_scores_give_mean_of_values():
    """q's latent part zero and all rope keys equal: every score equals s, so
    o = mean of the value rows and lse = s + ln L."""
    wl = W.make_case([77], h=4, seed=6)
    wl.q[..., :512] = 0
    kv = wl.kv_cache.reshape(-1, 576)
    kv[:, 512:] = kv[0, 512:]
    o, lse = run_oracle(wl)
    vals = _decode_kv(wl)
    slots = wl.req_to_token[int(wl.req_pool_indices[0]), :77].numpy()
    mean = vals[slots, :512].mean(axis=0)
    s = wl.softmax_scale * (wl.q[0, 0].to(torch.float64).numpy() @ vals[slots[0]])
    assert np.allclose(o[0, 0], mean, atol=1e-12)
    assert np.allclose(lse[0, 0], s + math.log(77), atol=1e-12)


def test_two_keys_log3_gap():
    """Two keys whose scores differ by exactly ln 3 in value: weights 3/4 and 1/4."""
    wl = W.make_case([2], h=1, seed=8)
    wl.q.zero_()
    wl.q[0, 0, 0, 0] = 1.0
    kv = wl.kv_cache.reshape(-1, 576)
    slots = wl.req_to_token[int(wl.req_pool_indices[0]), :2].numpy()
    kv[slots[0], 0] = 4.0
    kv[slots[1], 0] = 2.0
    # scores 4*scale and 2*scale; choose scale so the gap is ln 3
    wl.softmax_scale = math.log(3.0) / 2.0
    o, lse = run_oracle(wl)
    v = _decode_kv(wl)
    expect = 0.75 * v[slots[0], :512] + 0.25 * v[slots[1], :512]
    assert np.allclose(o[0, 0, 0], expect, atol=1e-12)
    s0 = 4.0 * wl.softmax_scale
    assert math.isclose(lse[0, 0, 0], s0 + math.log(4.0 / 3.0), abs_tol=1e-12)


def test_large_scores_are_stable():
    wl = W.make_case([150, 40], h=4, seed=9)
    wl.q.mul_(200.0)
    o, lse = run_oracle(wl)
    bo, blse = brute_force(wl)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    assert np.allclose(o, bo, rtol=1e-10, atol=1e-10)
    assert np.allclose(lse, blse, rtol=1e-12, atol=1e-9)


def test_page_permutation_invariance():
    wl = W.make_case([130, 64, 7], h=4, seed=10, pool_factor=2.0)
    o1, l1 = run_oracle(wl)
    n_pages = wl.kv_cache.shape[0]
    perm = torch.from_numpy(np.random.default_rng(1).permutation(n_pages))
    kv2 = torch.empty_like(wl.kv_cache)
    kv2[perm] = wl.kv_cache
    r2t = wl.req_to_token.clone()
    r2t = perm[r2t // 64].to(torch.int32) * 64 + r2t % 64
    wl.kv_cache, wl.req_to_token = kv2, r2t
    o2, l2 = run_oracle(wl)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


@pytest.mark.parametrize("causal", [True, False])
def test_split_then_merge_equals_unsplit(causal):
    wl = W.make_case([300, 129, 64], h=3, q_len=2, verify=True, seed=12)
    o, lse = run_oracle(wl, causal=causal)
    rng = np.random.default_rng(4)
    bs, q_len, h = 3, 2, 3
    L = wl.cache_seqlens.numpy().astype(np.int64)
    cuts = [np.sort(rng.integers(0, L[b] + 1, 3)) for b in range(bs)]
    bounds = [np.concatenate([[0], c, [L[b]]]) for b, c in enumerate(cuts)]
    parts = []
    for k in range(4):
        kb = np.array([bounds[b][k] for b in range(bs)])
        ke = np.array([bounds[b][k + 1] for b in range(bs)])
        parts.append(run_oracle(wl, causal=causal, key_begin=kb, key_end=ke))
    for b in range(bs):
        for i in range(q_len):
            for hh in range(h):
                op = np.stack([p[0][b, i, hh] for p in parts])
                lp = np.array([p[1][b, i, hh] for p in parts])
                om, lm = oracle.merge_states(op, lp)
                assert np.allclose(om, o[b, i, hh], atol=1e-12)
                assert math.isclose(lm, lse[b, i, hh], abs_tol=1e-12)


def test_verify_query_equals_shorter_decode():
    wl = W.make_case([90, 200], h=4, q_len=4, verify=True, seed=13)
    o, lse = run_oracle(wl)
    for i in range(4):
        dec = W.Workload(**{**wl.__dict__})
        dec.q = wl.q[:, i:i + 1].clone()
        dec.cache_seqlens = wl.cache_seqlens - 4 + 1 + i
        od, ld = run_oracle(dec)
        assert np.array_equal(od[:, 0], o[:, i]) and np.array_equal(ld[:, 0], lse[:, i])


def test_heads_are_independent():
    wl = W.make_case([150, 20], h=6, seed=14)
    o, lse = run_oracle(wl)
    one = W.Workload(**{**wl.__dict__})
    one.q = wl.q[:, :, 4:5].clone()
    o1, l1 = run_oracle(one)
    assert np.array_equal(o1[:, :, 0], o[:, :, 4]) and np.array_equal(l1[:, :, 0], lse[:, :, 4])


def test_fp8_equals_bf16_on_dequantized_cache():
    """With a power-of-two descale every dequantized e4m3 value is exact in bf16, so
    the fp8 oracle must equal the bf16 oracle on the dequantized cache."""
    wl = W.make_case([100, 65], h=4, kv="fp8", seed=15)
    wl.descale_k = torch.tensor([0.0078125])
    o8, l8 = run_oracle(wl)
    deq = (wl.kv_cache.to(torch.float64) * 0.0078125).to(torch.bfloat16)
    assert torch.equal(deq.to(torch.float64), wl.kv_cache.to(torch.float64) * 0.0078125)
    b16 = W.Workload(**{**wl.__dict__})
    b16.kv_cache, b16.descale_k, b16.descale_q = deq, None, None
    ob, lb = run_oracle(b16)
    assert np.array_equal(o8, ob) and np.array_equal(l8, lb)


def test_e5m2_cache_equals_bf16_on_dequantized_cache():
    """An e5m2 cache (the other fp8 format the backend accepts) with its descale equals the
    bf16 oracle on a cache holding the dequantised values (e5m2 x scale is exact in bf16
    for a power-of-two scale)."""
    wl = W.make_case([100, 37], h=8, seed=12)
    codes = (wl.kv_cache.float() * 4).to(torch.float8_e5m2)
    scale = 0.25
    deq = (codes.float() * scale).to(torch.bfloat16)
    assert torch.equal(deq.float(), codes.float() * scale)
    o8, l8 = oracle.mla_decode(wl.q, codes, wl.req_to_token, wl.req_pool_indices, wl.cache_seqlens,
                               wl.softmax_scale, True, kv_is_fp8=True, descale_k=scale)
    ob, lb = oracle.mla_decode(wl.q, deq, wl.req_to_token, wl.req_pool_indices, wl.cache_seqlens,
                               wl.softmax_scale, True)
    assert np.allclose(o8, ob, rtol=0, atol=1e-12) and np.allclose(l8, lb, rtol=0, atol=1e-12)


def test_fp8_query_equals_bf16_query_on_its_values():
    """A query given as e4m3 codes (the FlashMLA backend page quantises q with
    scaled_fp8_quant before the call, descale_q being the scale): every e4m3 value is exact in
    bf16, so the oracle on the codes must equal the oracle on a bf16 q holding their values,
    with the same descale_q, on a bf16 and on an e4m3 cache."""
    for kv in ("bf16", "fp8"):
        wl = W.make_case([90, 200, 1], h=4, kv=kv, seed=18)
        scale = 0.03125
        codes = (wl.q.to(torch.float32) / scale).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
        vals = codes.to(torch.bfloat16)
        assert torch.equal(vals.to(torch.float64), codes.to(torch.float64))
        dk = float(wl.descale_k[0]) if wl.descale_k is not None else 1.0
        args = (wl.kv_cache, wl.req_to_token, wl.req_pool_indices, wl.cache_seqlens, wl.softmax_scale,
                wl.causal)
        o8, l8 = oracle.mla_decode(codes, *args, kv_is_fp8=wl.is_fp8, descale_q=scale, descale_k=dk,
                                   q_is_fp8=True)
        ob, lb = oracle.mla_decode(vals, *args, kv_is_fp8=wl.is_fp8, descale_q=scale, descale_k=dk)
        assert np.array_equal(o8, ob) and np.array_equal(l8, lb)
        # and the scale really enters: descale_q = 2 * scale doubles every score
        o2, l2 = oracle.mla_decode(codes, *args, kv_is_fp8=wl.is_fp8, descale_q=2 * scale,
                                   descale_k=dk, q_is_fp8=True)
        assert not np.allclose(l2, l8)


def test_empty_and_fully_masked_rows():
    wl = W.make_case([0, 3], h=2, seed=16)
    o, lse = run_oracle(wl)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(lse[1]))
    # verify with cache length shorter than q_len: early draft rows see no key
    wl = W.make_case([0], h=2, q_len=3, verify=True, seed=17)
    wl.cache_seqlens[0] = 2
    o, lse = run_oracle(wl)
    assert np.all(o[0, 0] == 0) and np.all(np.isneginf(lse[0, 0]))
    assert np.all(np.isfinite(lse[0, 1:]))


def test_merge_states_closed_forms():
    rng = np.random.default_rng(0)
    a, b = rng.standard_normal(8), rng.standard_normal(8)
    o, l = oracle.merge_states(np.stack([a, b]), np.array([1.5, 1.5]))
    assert np.allclose(o, (a + b) / 2, atol=1e-15) and math.isclose(l, 1.5 + math.log(2))
    o, l = oracle.merge_states(np.stack([a, b]), np.array([-np.inf, 0.25]))
    assert np.array_equal(o, b) and l == 0.25
    o, l = oracle.merge_states(np.stack([a, b]), np.array([-np.inf, -np.inf]))
    assert np.all(o == 0) and l == -np.inf
    o, l = oracle.merge_states(np.stack([a, b]), np.array([0.0, math.log(3.0)]))
    assert np.allclose(o, 0.25 * a + 0.75 * b, atol=1e-15)
    assert math.isclose(l, math.log(4.0), abs_tol=1e-15)
