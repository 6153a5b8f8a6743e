"""The C-ABI library builds for sm_100a, loads without a GPU, exports every symbol the
header declares, and its host-only logic (part count, workspace size, argument
validation) behaves as documented.  No call here reaches a CUDA API."""
import ctypes
import os
import re

import pytest

import oracle
import paged_kv_mla_create_b200 as mla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla_b200.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = mla.library()
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n


def test_abi_version_and_status_strings():
    lib = mla.library()
    assert lib.mla_abi_version() == 2
    for code, name in mla._STATUS.items():
        assert lib.mla_status_string(code).decode() == name


@pytest.mark.parametrize("sm,heads,hk", [(148, 128, 1), (148, 512, 1), (148, 16, 1), (148, 129, 1),
                                         (132, 128, 1), (1, 128, 1), (148, 128, 2), (148, 4096, 1)])
def test_num_sm_parts_matches_oracle(sm, heads, hk):
    assert mla.library().mla_num_sm_parts(sm, heads, hk) == oracle.num_sm_parts(sm, heads, hk)


def test_num_sm_parts_rejects_bad_arguments():
    lib = mla.library()
    assert lib.mla_num_sm_parts(0, 128, 1) == -1
    assert lib.mla_num_sm_parts(148, 0, 1) == -1
    assert lib.mla_num_sm_parts(148, 128, 0) == -1


def test_workspace_bytes():
    lib = mla.library()
    ws = lib.mla_decode_workspace_bytes(64, 1, 128, 74)
    rows, splits = 128, 64 + 74
    a256 = lambda x: -(-x // 256) * 256
    # arrival words [bs, query tiles, 2] int32, then the partials and their lse
    expect = a256(64 * 1 * 2 * 4) + a256(splits * rows * 512 * 4) + a256(splits * rows * 4)
    assert ws == expect
    ws4 = lib.mla_decode_workspace_bytes(32, 4, 128, 18)
    assert ws4 == a256(32 * 4 * 2 * 4) + a256(50 * 512 * 512 * 4) + a256(50 * 512 * 4)
    assert lib.mla_decode_workspace_bytes(0, 1, 128, 74) == 0
    assert lib.mla_decode_workspace_bytes(1, 1, 128, 0) == 0


def _decode(lib, **over):
    args = dict(q=1 << 20, q_dtype=0, bs=2, q_len=1, h_q=16, head_dim=576, head_dim_v=512,
                k_cache=1 << 21, kv_dtype=0, num_pages=8, page_size=64, block_table=1 << 22,
                bt_stride=3, max_pages=3, cache_seqlens=1 << 23, md=1 << 24, parts=74,
                num_splits=1 << 25, scale=0.07, causal=1, dq=None, dk=None, out=1 << 26,
                lse=1 << 27, ws=1 << 28, ws_bytes=1 << 30, stream=None)
    args.update(over)
    return lib.mla_decode_paged(*args.values())


def test_decode_validation_happens_before_any_launch():
    lib = mla.library()
    assert _decode(lib, bs=0) == 0                       # idle batch: nothing to do
    assert _decode(lib, head_dim=512) == 2               # unsupported head dims
    assert _decode(lib, head_dim_v=576) == 2
    assert _decode(lib, page_size=32) == 2
    assert _decode(lib, q_dtype=1) == 2                  # e4m3 q needs an e4m3 cache
    assert _decode(lib, q_dtype=1, kv_dtype=4) == 2      # ... not e5m2
    assert _decode(lib, q_dtype=3) == 1                  # not a query type
    assert _decode(lib, kv_dtype=7) == 1
    assert _decode(lib, causal=2) == 1
    assert _decode(lib, q=None) == 1
    assert _decode(lib, num_pages=0) == 1
    assert _decode(lib, num_pages=1 << 26) == 1          # 64 * pages must fit int32 rows
    assert _decode(lib, max_pages=4) == 1                # stride smaller than max_pages
    assert _decode(lib, q=(1 << 20) + 8) == 1            # misaligned q
    assert _decode(lib, ws_bytes=16) == 5                # workspace too small
    assert _decode(lib, ws=None) == 5
    assert _decode(lib, scale=float("nan")) == 1
    assert _decode(lib, dk=1 << 29) == 1                 # descale_k with a bf16 cache
    assert _decode(lib, q_len=1, h_q=65535 * 128 + 1) == 2   # more query tiles than grid.y holds


def test_test_hooks_validation():
    lib = mla.library()
    assert lib.mla_set_test_hooks(0, -2, 0) == 1
    assert lib.mla_set_test_hooks(0, -1, 0) == 0     # the defaults (no launch involved)


def test_set_kv_buffer_validation():
    lib = mla.library()
    kv = lib.mla_set_kv_buffer
    ok = dict(pool=1 << 20, dt=1, slots=100, loc=1 << 21, loc_dt=3, n=4, k=1 << 22, stride=576,
              scale=None, stream=None)
    assert kv(*{**ok, "n": 0}.values()) == 0                 # nothing to write
    assert kv(*{**ok, "dt": 9}.values()) == 1
    assert kv(*{**ok, "loc_dt": 0}.values()) == 1
    assert kv(*{**ok, "dt": 0, "scale": 1 << 23}.values()) == 1   # a scale is for fp8 pools
    assert kv(*{**ok, "stride": 570}.values()) == 1
    assert kv(*{**ok, "stride": 580}.values()) == 1          # not a multiple of 8
    assert kv(*{**ok, "k": (1 << 22) + 8}.values()) == 1     # misaligned k
    assert kv(*{**ok, "pool": None}.values()) == 1
    assert kv(*{**ok, "n": -1}.values()) == 1


def test_block_table_and_planner_validation():
    lib = mla.library()
    bt = lib.mla_build_block_table
    ok = dict(r2t=1 << 20, rows=5, stride=192, rpi=1 << 21, rpi_dt=3, sl=1 << 22, sl_dt=2, add=0,
              bs=2, out=1 << 23, out_stride=3, max_pages=3, page=64, fill=1, stream=None)
    assert bt(*{**ok, "bs": 0}.values()) == 0
    assert bt(*{**ok, "page": 16}.values()) == 1
    assert bt(*{**ok, "rpi_dt": 0}.values()) == 1
    assert bt(*{**ok, "out_stride": 2}.values()) == 1
    assert bt(*{**ok, "r2t": None}.values()) == 1
    md = lib.mla_get_mla_metadata
    # (cache_seqlens, bs, num_heads_per_head_k, num_heads_k, is_fp8, sm_count, md, ns, stream)
    assert md(1 << 20, 2, 0, 1, 0, 148, 1 << 21, 1 << 22, None) == 1     # no heads
    assert md(1 << 20, 2, 128, 0, 0, 148, 1 << 21, 1 << 22, None) == 1   # no KV heads
    assert md(1 << 20, 2, 128, 1, 0, 0, 1 << 21, 1 << 22, None) == 1     # no SMs
    assert md(1 << 20, -1, 128, 1, 0, 148, 1 << 21, 1 << 22, None) == 1
    assert md(1 << 20, 2, 128, 1, 0, 148, (1 << 21) + 4, 1 << 22, None) == 1   # misaligned rows
    assert md(1 << 20, 2, 128, 1, 0, 148, None, 1 << 22, None) == 1
    dm = lib.mla_build_decode_metadata
    okm = dict(r2t=1 << 20, rows=5, stride=192, rpi=1 << 21, rpi_dt=3, sl=1 << 22, sl_dt=2, add=0,
               bs=2, out=1 << 23, out_stride=3, max_pages=3, page=64, fill=1, heads=128, hk=1,
               fp8=0, sms=148, cl=None, md=1 << 24, ns=1 << 25, stream=None)
    assert dm(*{**okm, "page": 32}.values()) == 1
    assert dm(*{**okm, "sms": 0}.values()) == 1
    assert dm(*{**okm, "heads": 0}.values()) == 1
    assert dm(*{**okm, "sl_dt": 0}.values()) == 1
    assert dm(*{**okm, "md": (1 << 24) + 4}.values()) == 1
    assert dm(*{**okm, "r2t": None}.values()) == 1
    assert dm(*{**okm, "out_stride": 2}.values()) == 1


def test_merge_state_validation():
    lib = mla.library()
    ms = lib.mla_merge_state
    ok = dict(oa=1 << 20, la=1 << 21, ob=1 << 22, lb=1 << 23, rows=8, dv=512, o=1 << 24, lse=1 << 25, stream=None)
    assert ms(*{**ok, "rows": 0}.values()) == 0              # nothing to merge
    assert ms(*{**ok, "rows": -1}.values()) == 1
    assert ms(*{**ok, "dv": 256}.values()) == 2
    assert ms(*{**ok, "oa": None}.values()) == 1
    assert ms(*{**ok, "lse": None}.values()) == 1
    assert ms(*{**ok, "ob": (1 << 22) + 8}.values()) == 1   # misaligned o_b


def test_extend_workspace_bytes():
    """The extend workspace: a padded copy of the new rows (when e is not a multiple of 64),
    then for each part a page table, lengths, plan, an attention workspace and the partial
    result, every piece 256-byte aligned."""
    lib = mla.library()
    a256 = lambda x: -(-x // 256) * 256
    for bs, e, h, mpp, sm in [(2, 37, 16, 4, 148), (3, 64, 128, 10, 148), (1, 1, 128, 0, 132)]:
        parts = oracle.num_sm_parts(sm, e * h, 1)
        e_pad = -(-e // 64) * 64
        rows = bs * e * h
        ws = lib.mla_decode_workspace_bytes(bs, e, h, parts)
        pool = bs * e_pad * 576 * 2 if e_pad != e else 0
        part = lambda pages: (a256(bs * pages * 4) + a256(bs * 4) + a256(parts * 32) + a256((bs + 1) * 4) + a256(ws)
                              + a256(rows * 1024) + a256(rows * 4))
        assert lib.mla_extend_workspace_bytes(bs, e, h, mpp, sm) == a256(pool) + part(e_pad // 64) + part(max(mpp, 1))
    assert lib.mla_extend_workspace_bytes(0, 37, 16, 4, 148) == 0
    assert lib.mla_extend_workspace_bytes(2, 0, 16, 4, 148) == 0
    assert lib.mla_extend_workspace_bytes(2, 37, 16, -1, 148) == 0
    assert lib.mla_extend_workspace_bytes(2, 37, 16, 4, 0) == 0


def test_extend_validation_happens_before_any_launch():
    lib = mla.library()
    ex = lib.mla_extend_paged_prefix
    ok = dict(q=1 << 20, bs=2, e=37, h=16, k_new=1 << 21, kv=1 << 22, kv_dt=0, pages=8, r2t=1 << 23, rows=5,
              stride=512, rpi=1 << 24, rpi_dt=3, pl=1 << 25, mpp=4, scale=0.07, dk=None, sm=148, out=1 << 26,
              lse=1 << 27, ws=1 << 28, ws_bytes=16, stream=None)
    assert ex(*{**ok, "bs": 0}.values()) == 0                # idle batch
    assert ex(*{**ok, "e": 0}.values()) == 1
    assert ex(*{**ok, "h": 0}.values()) == 1
    assert ex(*{**ok, "sm": 0}.values()) == 1
    assert ex(*{**ok, "mpp": -1}.values()) == 1
    assert ex(*{**ok, "q": None}.values()) == 1
    assert ex(*{**ok, "pl": None}.values()) == 1
    assert ex(*{**ok, "k_new": (1 << 21) + 8}.values()) == 1   # misaligned new rows
    assert ex(*{**ok, "e": 65535, "h": 129}.values()) == 2     # more query rows than the kernel's grid holds
    assert ex(*ok.values()) == 5                               # workspace too small
    assert ex(*{**ok, "ws": None}.values()) == 5
