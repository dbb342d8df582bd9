"""Seeded synthetic workloads for paged latent (MLA) attention.

Recipe (the same for every config):
  * one CPU ``torch.Generator`` seeded with ``seed`` (0 unless stated);
  * draw order: kv lengths -> page assignment (a random permutation of the page
    pool) -> q_nope -> q_pe -> cache;
  * every value ``randn * 0.5`` (standard deviation 0.5), rounded to bf16;
  * the pool holds exactly the pages the rows need (plus any stated extra), and
    the page table is a random permutation of it;
  * rows sharing a prefix name the same physical pages for it.

The five named workloads follow the configurations the latent-attention
benchmark is quoted on: tiny decode, batch-64 decode, long-context decode,
a mixed chunked-prefill step, and speculative decode with shared prefixes.
Nothing here computes attention: only lengths, page tables and random tensors.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

KV_LORA_RANK = 512
ROPE_DIM = 64
LATENT = KV_LORA_RANK + ROPE_DIM
SM_SCALE = 192 ** -0.5  # softmax scale of the original 192-wide query/key head

CONFIG_NAMES = (
    "tiny_decode",
    "decode_b64",
    "long_decode",
    "mixed_prefill",
    "spec_shared_prefix",
)


@dataclasses.dataclass
class MlaInputs:
    name: str
    num_heads: int
    page_size: int
    num_pages: int
    causal: bool
    return_lse: bool
    sm_scale: float
    qo_indptr: torch.Tensor  # int32 [B+1]
    kv_indptr: torch.Tensor  # int32 [B+1]
    kv_indices: torch.Tensor  # int32 [sum n_b]
    last_page_len: torch.Tensor  # int32 [B]
    q_nope: torch.Tensor  # bf16 [T, H, 512]
    q_pe: torch.Tensor  # bf16 [T, H, 64]
    cache: torch.Tensor  # bf16 [num_pages, page_size, 576]
    q_lens: list
    kv_lens: list
    description: str = ""

    @property
    def batch(self) -> int:
        return len(self.q_lens)

    @property
    def total_tokens(self) -> int:
        return int(self.qo_indptr[-1])

    def to(self, device) -> "MlaInputs":
        d = dataclasses.replace(self)
        d.q_nope = self.q_nope.to(device)
        d.q_pe = self.q_pe.to(device)
        d.cache = self.cache.to(device)
        return d


def _randn_bf16(shape, gen, std=0.5, chunk_elems=1 << 26) -> torch.Tensor:
    """randn * std rounded to bf16, drawn in chunks so large caches do not need a
    full float32 temporary."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.bfloat16)
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        out[s:e] = (torch.randn(e - s, generator=gen) * std).to(torch.bfloat16)
    return out.view(*shape)


def make_custom(
    q_lens: Sequence[int],
    kv_lens: Sequence[int],
    num_heads: int,
    page_size: int,
    *,
    seed: int = 0,
    causal: bool = True,
    return_lse: bool = True,
    extra_pool_pages: int = 0,
    shared_group: int = 0,
    shared_pages: int = 0,
    std: float = 0.5,
    name: str = "custom",
    gen: Optional[torch.Generator] = None,
    pool_pages: Optional[int] = None,
    tables_only: bool = False,
) -> MlaInputs:
    """Build one seeded workload from explicit per-row query and key counts.

    ``shared_group`` rows in a row (0 = none) name the same first ``shared_pages``
    physical pages (a shared prefix); every other page is unique to its row.
    ``pool_pages`` (if given) fixes the pool size; the pages are then drawn as a
    random subset of it (``randperm(pool)[:needed]``).  ``tables_only`` skips the
    random tensors (they are drawn last, so the tables are the same either way).
    """
    if gen is None:
        gen = torch.Generator().manual_seed(seed)
    B = len(q_lens)
    assert len(kv_lens) == B
    n_pages = [(-(-int(k) // page_size)) for k in kv_lens]
    last = [int(k) - (n - 1) * page_size if n > 0 else 1 for k, n in zip(kv_lens, n_pages)]

    # page assignment
    if shared_group and shared_pages:
        n_groups = -(-B // shared_group)
        for b in range(B):
            assert n_pages[b] >= shared_pages, "shared prefix longer than a row"
        needed = n_groups * shared_pages + sum(n - shared_pages for n in n_pages)
    else:
        needed = sum(n_pages)
    if pool_pages is None:
        pool = needed + extra_pool_pages
        perm = torch.randperm(pool, generator=gen)
    else:
        pool = pool_pages
        assert pool >= needed
        perm = torch.randperm(pool, generator=gen)
    cursor = 0
    indices = []
    shared_ids = {}
    for b in range(B):
        row = []
        if shared_group and shared_pages:
            g = b // shared_group
            if g not in shared_ids:
                shared_ids[g] = perm[cursor : cursor + shared_pages].tolist()
                cursor += shared_pages
            row.extend(shared_ids[g])
            own = n_pages[b] - shared_pages
        else:
            own = n_pages[b]
        row.extend(perm[cursor : cursor + own].tolist())
        cursor += own
        indices.extend(row)

    qo = [0]
    for q in q_lens:
        qo.append(qo[-1] + int(q))
    kvp = [0]
    for n in n_pages:
        kvp.append(kvp[-1] + n)
    T = qo[-1]
    if tables_only:
        q_nope = q_pe = cache = None
    else:
        q_nope = _randn_bf16((T, num_heads, KV_LORA_RANK), gen, std)
        q_pe = _randn_bf16((T, num_heads, ROPE_DIM), gen, std)
        cache = _randn_bf16((pool, page_size, LATENT), gen, std)
    return MlaInputs(
        name=name,
        num_heads=num_heads,
        page_size=page_size,
        num_pages=pool,
        causal=causal,
        return_lse=return_lse,
        sm_scale=SM_SCALE,
        qo_indptr=torch.tensor(qo, dtype=torch.int32),
        kv_indptr=torch.tensor(kvp, dtype=torch.int32),
        kv_indices=torch.tensor(indices, dtype=torch.int32),
        last_page_len=torch.tensor(last, dtype=torch.int32),
        q_nope=q_nope,
        q_pe=q_pe,
        cache=cache,
        q_lens=[int(q) for q in q_lens],
        kv_lens=[int(k) for k in kv_lens],
    )


def _randint(lo: int, hi: int, n: int, gen) -> list:
    """n integers uniform on the closed range [lo, hi]."""
    return torch.randint(lo, hi + 1, (n,), generator=gen).tolist()


def make_config(name: str, seed: int = 0, tables_only: bool = False) -> MlaInputs:
    """One of the five named workloads (see module docstring), seeded."""
    gen = torch.Generator().manual_seed(seed)
    kw = dict(gen=gen, name=name, tables_only=tables_only)
    if name == "tiny_decode":
        d = make_custom([1, 1], [37, 150], 16, 16, causal=True, return_lse=True, pool_pages=32, **kw)
        d.description = ("2 rows, q_len 1, kv lens 37 and 150, H=16, page_size 16, 13 pages "
                         "drawn from a permuted 32-page pool, lse on")
        return d
    if name == "decode_b64":
        kv = _randint(512, 8192, 64, gen)
        d = make_custom([1] * 64, kv, 128, 64, causal=True, return_lse=False, **kw)
        d.description = "64 rows, q_len 1, kv ~ U{512..8192}, H=128, page_size 64, shuffled pool, lse off"
        return d
    if name == "long_decode":
        d = make_custom([1] * 16, [32768] * 16, 128, 64, causal=True, return_lse=True, **kw)
        d.description = "16 rows, q_len 1, kv 32768, H=128, page_size 64, lse on"
        return d
    if name == "mixed_prefill":
        kv_dec = _randint(1024, 4096, 60, gen)
        q = [1024] * 4 + [1] * 60
        kv = [2048 + 1024] * 4 + kv_dec
        d = make_custom(q, kv, 128, 64, causal=True, return_lse=False, **kw)
        d.description = ("4 prefill rows (1024 new tokens after a 2048-token prefix, causal "
                         "end-aligned) + 60 decode rows kv ~ U{1024..4096}; H=128, page_size 64")
        return d
    if name == "spec_shared_prefix":
        kv = _randint(1024, 16384, 128, gen)
        d = make_custom([4] * 128, kv, 128, 64, causal=True, return_lse=True, shared_group=8,
                        shared_pages=16, **kw)
        d.description = ("128 rows, q_len 4 (causal, end-aligned), kv ~ U{1024..16384}, groups of 8 "
                         "rows share their first 1024 tokens of pages; H=128, page_size 64, lse on")
        return d
    raise KeyError(name)
