"""Seeded synthetic inputs for paged MLA decode.

This module only draws inputs: random page permutations, request lengths, normal
query and latent-KV values, and the per-tensor e4m3 quantisation of the cache that
an upstream KV writer would have produced.  It holds none of the attention,
page-table or planning arithmetic, so both the CUDA path and the CPU oracle can be
fed from it without sharing any of the method.

Layouts follow the SGLang FlashMLA attention backend page (flashmla_backend.py):
``q`` is ``[bs, q_len, h, 576]`` (kv_lora_rank 512 + qk_rope_head_dim 64), the KV
pool is a token-slot buffer viewed ``[-1, 64, 1, 576]`` (stored here as
``[num_pages, 64, 576]``), ``req_to_token`` maps (request-pool row, position) to a
token slot, and target-verify appends ``num_draft_tokens`` (= q_len) positions to
each request before attention.

Pool recipe: each request owns cdiv(L, 64) whole pages drawn without replacement
from a shuffled pool of ceil(1.25 * pages needed) pages (exactly 8 for the tiny
case); token slots run in order inside a page, so the slot of position j is
64 * page + j % 64.  ``req_to_token`` has bs + 3 rows and ``req_pool_indices`` is a
random choice of distinct rows.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

PAGE = 64
D_QK = 576
D_V = 512
SOFTMAX_SCALE = 1.0 / math.sqrt(192.0)
POISON = 3.0e4          # finite poison for unused pages / tail rows (bf16 rounds it to 29952)
POISON_FP8 = 448.0      # largest finite e4m3 value
POISON_E5M2 = 57344.0   # largest finite e5m2 value


@dataclasses.dataclass
class Workload:
    name: str
    q: torch.Tensor                 # bf16, or e4m3 codes, [bs, q_len, h, 576]
    kv_cache: torch.Tensor          # bf16 or float8_e4m3fn [num_pages, 64, 576]
    req_to_token: torch.Tensor      # int32 [bs + 3, max_ctx]
    req_pool_indices: torch.Tensor  # int64 [bs]
    seq_lens: torch.Tensor          # int32 [bs]  (prefix lengths in target-verify)
    cache_seqlens: torch.Tensor     # int32 [bs]  (seq_lens + num_draft_tokens in verify)
    num_draft_tokens: int           # 0 in decode, q_len in target-verify
    softmax_scale: float
    causal: bool
    descale_q: Optional[torch.Tensor]  # fp32 [1] (fp8 cache only): the scale q was quantised with
    descale_k: Optional[torch.Tensor]  # fp32 [1] (fp8 cache only)

    @property
    def bs(self) -> int:
        return int(self.q.shape[0])

    @property
    def q_len(self) -> int:
        return int(self.q.shape[1])

    @property
    def h(self) -> int:
        return int(self.q.shape[2])

    @property
    def is_fp8(self) -> bool:
        return self.kv_cache.dtype in (torch.float8_e4m3fn, torch.float8_e5m2)

    @property
    def q_is_fp8(self) -> bool:
        return self.q.dtype == torch.float8_e4m3fn

    @property
    def max_pages(self) -> int:
        lmax = int(self.cache_seqlens.max()) if self.bs else 0
        return max(1, -(-lmax // PAGE))

    def to(self, device) -> "Workload":
        kw = {}
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            kw[f.name] = v.to(device) if isinstance(v, torch.Tensor) else v
        return Workload(**kw)


# The five workloads: (name, bs, h, q_len, length recipe, kv dtype).
CONFIGS = {
    1: dict(name="tiny MLA decode (bs 2, L {37,130}, h 16)", bs=2, h=16, q_len=1,
            lengths=("fixed", [37, 130]), kv="bf16", pool_pages=8),
    2: dict(name="DeepSeek-V3-shaped decode (bs 64, h 128, L~U[1024,4096], bf16)", bs=64, h=128,
            q_len=1, lengths=("uniform", 1024, 4096), kv="bf16"),
    3: dict(name="skewed long-context decode (bs 8, h 128, 1x131072 + 7xU[512,2048], bf16)", bs=8,
            h=128, q_len=1, lengths=("skewed", 131072, 512, 2048), kv="bf16"),
    4: dict(name="fp8 KV decode (bs 128, h 128, L 4096, e4m3 per-tensor scale)", bs=128, h=128,
            q_len=1, lengths=("fixed", [4096] * 128), kv="fp8"),
    5: dict(name="target-verify (bs 32, h 128, q_len 4, prefix~U[2048,8192], bf16)", bs=32,
            h=128, q_len=4, lengths=("uniform", 2048, 8192), kv="bf16", verify=True),
}


def _draw_lengths(rng: np.random.Generator, recipe, bs: int) -> List[int]:
    kind = recipe[0]
    if kind == "fixed":
        return [int(x) for x in recipe[1]]
    if kind == "uniform":
        return [int(x) for x in rng.integers(recipe[1], recipe[2] + 1, size=bs)]
    if kind == "skewed":
        return [int(recipe[1])] + [int(x) for x in rng.integers(recipe[2], recipe[3] + 1,
                                                                 size=bs - 1)]
    raise ValueError(kind)


def make_case(seq_lens: List[int], h: int, q_len: int = 1, kv: str = "bf16",
              verify: bool = False, seed: int = 0, poison: bool = False,
              pool_pages: Optional[int] = None, name: str = "custom",
              pool_factor: float = 1.25, q_fp8: bool = False) -> Workload:
    """Draw one workload.  seq_lens are prefix lengths; in target-verify each request
    gets q_len more positions (the draft tokens) before attention.  With an fp8 cache,
    q_fp8 hands q over as e4m3 codes the way the FlashMLA backend page's fp8 branch does:
    quantised with the cache's own scale (q_scale = k_scale), saturating at +-448, with
    descale_q = that scale."""
    rng = np.random.default_rng(seed)
    bs = len(seq_lens)
    n_draft = q_len if verify else 0
    cache_lens = [int(s) + n_draft for s in seq_lens]
    pages_per_req = [-(-L // PAGE) for L in cache_lens]
    need = sum(pages_per_req)
    if pool_pages is None:
        pool_pages = max(1, int(math.ceil(pool_factor * need)))
    if pool_pages < need:
        raise ValueError("pool too small")
    perm = rng.permutation(pool_pages)
    rows = bs + 3
    max_ctx = max(1, max(pages_per_req, default=1)) * PAGE
    req_to_token = np.zeros((rows, max_ctx), dtype=np.int32)
    rpi = rng.permutation(rows)[:bs].astype(np.int64)
    owned = []
    cursor = 0
    for b in range(bs):
        pages = perm[cursor:cursor + pages_per_req[b]]
        cursor += pages_per_req[b]
        owned.append(pages)
        if len(pages):
            slots = (pages[:, None] * PAGE + np.arange(PAGE)[None, :]).reshape(-1)
            req_to_token[rpi[b], :slots.shape[0]] = slots
    q = torch.from_numpy(rng.standard_normal((bs, q_len, h, D_QK), dtype=np.float32))
    x = rng.standard_normal((pool_pages, PAGE, D_QK), dtype=np.float32)
    descale_q = descale_k = None
    marks = None
    if poison:
        # token rows that no request may read: unused pages and each last page's tail
        marks = np.ones((pool_pages, PAGE), dtype=bool)
        for b in range(bs):
            if len(owned[b]):
                marks[owned[b]] = False
                tail = cache_lens[b] - (len(owned[b]) - 1) * PAGE
                marks[owned[b][-1], tail:] = True
        signs = np.where(rng.random((int(marks.sum()), D_QK)) < 0.5, -1.0, 1.0)
        x[marks] = 0.0
    if q_fp8 and kv != "fp8":
        raise ValueError("e4m3 queries go with an e4m3 cache")
    if kv == "bf16":
        if poison:
            x[marks] = (signs * POISON).astype(np.float32)
        kv_cache = torch.from_numpy(x).to(torch.bfloat16)
    elif kv in ("fp8", "e5m2"):
        # per-tensor scale: the largest magnitude maps to the format's largest finite value
        top = POISON_FP8 if kv == "fp8" else POISON_E5M2
        amax = float(np.abs(x).max()) if x.size else 0.0
        scale = np.float32(amax / top) if amax > 0 else np.float32(1.0)
        y = (x / scale).astype(np.float32)
        if poison:
            y[marks] = (signs * top).astype(np.float32)
        kv_cache = torch.from_numpy(y).to(torch.float8_e4m3fn if kv == "fp8" else torch.float8_e5m2)
        descale_k = torch.tensor([float(scale)], dtype=torch.float32)
        descale_q = torch.ones(1, dtype=torch.float32)
        if q_fp8:
            qb = q.to(torch.bfloat16).float()
            q = (qb / float(scale)).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
            descale_q = torch.tensor([float(scale)], dtype=torch.float32)
    else:
        raise ValueError(kv)
    return Workload(
        name=name,
        q=q if q.dtype == torch.float8_e4m3fn else q.to(torch.bfloat16),
        kv_cache=kv_cache,
        req_to_token=torch.from_numpy(req_to_token),
        req_pool_indices=torch.from_numpy(rpi),
        seq_lens=torch.tensor(list(seq_lens), dtype=torch.int32),
        cache_seqlens=torch.tensor(cache_lens, dtype=torch.int32),
        num_draft_tokens=n_draft,
        softmax_scale=SOFTMAX_SCALE,
        causal=True,
        descale_q=descale_q,
        descale_k=descale_k,
    )


def make_workload(index: int, poison: bool = False, seed: Optional[int] = None,
                  q_fp8: bool = False) -> Workload:
    """One of the five configured workloads, seeded with 1000 + index (q_fp8: its queries as
    e4m3 codes, for the fp8-cache workload)."""
    cfg = CONFIGS[index]
    s = 1000 + index if seed is None else seed
    rng = np.random.default_rng(s)
    lengths = _draw_lengths(rng, cfg["lengths"], cfg["bs"])
    return make_case(lengths, cfg["h"], cfg["q_len"], cfg["kv"], cfg.get("verify", False),
                     seed=s + 7919, poison=poison, pool_pages=cfg.get("pool_pages"),
                     name=cfg["name"] + (", e4m3 q" if q_fp8 else ""), q_fp8=q_fp8)
