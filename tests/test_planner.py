"""Bit-exact bookkeeping of the host planner against the oracle's independent reading
of the page tables (kv_len, visibility, page mapping), on host-only plans."""

import numpy as np
import pytest

import paged_head_latent_mla_b200 as M
from oracle import mla_oracle as O
from workloads import CONFIG_NAMES, make_config, make_custom

SCALE = 192 ** -0.5


def plan_tables(d, **kw):
    return M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=d.num_heads,
                      page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, causal=d.causal,
                      host_only=True, **kw)


def check_layout(d, desc, num_sms=148):
    H, P = d.num_heads, d.page_size
    qo = d.qo_indptr.numpy().astype(np.int64)
    kvp = d.kv_indptr.numpy().astype(np.int64)
    B = len(qo) - 1
    k_oracle = O.kv_lengths(kvp, d.last_page_len.numpy(), P)
    assert np.array_equal(desc["kv_len"].astype(np.int64), k_oracle)

    work, merge = desc["work"], desc["merge"]
    info = desc["info"]
    assert info["num_work"] == len(work) and info["num_merge"] == len(merge)
    # token -> batch row
    row_of_token = np.repeat(np.arange(B), np.diff(qo))
    # coverage[t] = list of (key_begin, key_end) from items covering token t
    cover = [[] for _ in range(int(qo[-1]))]
    partial_seen = []
    for (q_row0, n_rows, page_base, kv_len, kb, ke, diag, partial) in work:
        assert q_row0 % H == 0 and n_rows % H == 0 and 0 < n_rows <= 128
        t0 = q_row0 // H
        ntok = n_rows // H
        b = row_of_token[t0]
        assert row_of_token[t0 + ntok - 1] == b, "a tile crosses batch rows"
        assert page_base == kvp[b]  # so key j -> kv_indices[page_base + j // P], slot j % P
        assert kv_len == k_oracle[b]
        assert kb % M.MLA_KEY_TILE == 0 and kb <= ke or (kb == 0 and ke == 0)
        q_b = qo[b + 1] - qo[b]
        i0 = t0 - qo[b]
        vis_hi = O.visible_keys(int(k_oracle[b]), int(q_b), int(i0 + ntok - 1), d.causal)
        assert ke <= vis_hi
        for tt in range(ntok):
            i = i0 + tt
            vis = O.visible_keys(int(k_oracle[b]), int(q_b), int(i), d.causal)
            # the kernel's rule: keys < clamp(diag + tt + 1, 0, kv_len)
            assert min(max(diag + tt + 1, 0), kv_len) == vis
            cover[t0 + tt].append((kb, ke))
        if partial >= 0:
            partial_seen.append(partial)
    # every visible key of every query is covered exactly once
    for t in range(int(qo[-1])):
        b = row_of_token[t]
        vis = O.visible_keys(int(k_oracle[b]), int(qo[b + 1] - qo[b]), int(t - qo[b]), d.causal)
        spans = sorted(cover[t])
        assert spans, f"token {t} uncovered"
        pos = 0
        for (kb, ke) in spans:
            if ke <= kb:
                continue
            assert kb == pos, f"token {t}: gap/overlap at {pos} vs {kb}"
            pos = ke
        assert pos >= vis and pos <= max(vis, spans[-1][1])
        # no key beyond the tile's vis_hi is ever used, and keys beyond vis are masked
    # partial slots: each used exactly once, grouped contiguously per merge record
    assert sorted(partial_seen) == list(range(info["num_partials"]))
    for (q_row0, n_rows, first, n) in merge:
        assert n >= 2
        items = [w for w in work if w[7] >= first and w[7] < first + n]
        assert len(items) == n
        assert all(w[0] == q_row0 and w[1] == n_rows for w in items)
        spans = sorted((w[4], w[5]) for w in items)
        for a, b2 in zip(spans, spans[1:]):
            assert a[1] == b2[0] and a[1] % M.MLA_KEY_TILE == 0
    return True


@pytest.mark.parametrize("name", CONFIG_NAMES)
def test_named_config_layout(name):
    d = make_config(name, tables_only=True)
    p = plan_tables(d)
    check_layout(d, M.mla_plan_describe(p))


@pytest.mark.parametrize("split", [-1, 64, 128, 192, 1024])
@pytest.mark.parametrize("H,P", [(16, 16), (32, 32), (64, 64), (128, 128), (128, 16)])
def test_custom_layouts(split, H, P):
    rng = np.random.default_rng(H * 1000 + P + split)
    B = 9
    q = rng.integers(0, 40, B).tolist()
    k = rng.integers(0, 700, B).tolist()
    q[0], k[0] = 5, 0  # empty row with queries
    q[1], k[1] = 30, 7  # more queries than keys
    for causal in (True, False):
        d = make_custom(q, k, H, P, causal=causal, tables_only=True, extra_pool_pages=3, seed=split + H)
        p = plan_tables(d, split_keys=split)
        desc = M.mla_plan_describe(p)
        check_layout(d, desc)
        if split > 0:
            for w in desc["work"]:
                assert w[5] - w[4] <= split


def test_shared_prefix_page_mapping_matches_oracle():
    d = make_custom([4] * 16, [1100 + 37 * i for i in range(16)], 128, 64, shared_group=8, shared_pages=16,
                    tables_only=True)
    kvp = d.kv_indptr.numpy()
    idx = d.kv_indices.numpy()
    # rows of a group name identical first 16 pages
    for g in range(2):
        first = [tuple(idx[kvp[b]:kvp[b] + 16]) for b in range(8 * g, 8 * g + 8)]
        assert len(set(first)) == 1
    p = plan_tables(d)
    desc = M.mla_plan_describe(p)
    check_layout(d, desc)
    # the kernel's page lookup (page_base + j // P) equals the oracle's key_location
    for w in desc["work"][:8]:
        b = int(np.searchsorted(kvp, w[2], side="right") - 1)
        for j in (w[4], w[5] - 1):
            if j < 0 or j >= w[3]:
                continue
            assert O.key_location(kvp, idx, 64, b, int(j)) == (int(idx[w[2] + j // 64]), int(j % 64))


def test_auto_split_balances_long_decode():
    d = make_config("long_decode", tables_only=True)
    desc = M.mla_plan_describe(plan_tables(d))
    lens = [w[5] - w[4] for w in desc["work"]]
    assert desc["info"]["num_merge"] == 16  # every long row is split
    assert max(lens) <= 32768 // 4
    # balanced: total key tiles over 74 pairs vs the largest item
    T = M.MLA_KEY_TILE
    assert max(lens) / T <= 2 * (sum(lens) / T) / 74 + 8


def test_no_split_for_small_decode():
    d = make_config("tiny_decode", tables_only=True)
    desc = M.mla_plan_describe(plan_tables(d))
    assert desc["info"]["num_merge"] == 0 and desc["info"]["num_work"] == 2
