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


def check_layout(d, desc, context_only=False):
    """Check a plan's work items, merge records and merge references against the
    oracle's reading of the tables: every visible key of every query is covered exactly
    once; an item's visibility rule reproduces the oracle's; partial results occupy
    disjoint workspace rows; and every token whose items are partials is combined by
    exactly one merge record that references each of them exactly once."""
    H, P = d.num_heads, d.page_size
    qo = d.qo_indptr.numpy().astype(np.int64)
    kvp = d.kv_indptr.numpy().astype(np.int64)
    idx = d.kv_indices.numpy()
    B = len(qo) - 1
    k_full = O.kv_lengths(kvp, d.last_page_len.numpy(), P)
    q_len = np.diff(qo)
    k_att = k_full - q_len if context_only else k_full  # keys the queries attend
    assert np.array_equal(desc["kv_len"].astype(np.int64), k_att)
    causal = d.causal and not context_only

    def vis_of(b, i):
        return O.visible_keys(int(k_att[b]), int(q_len[b]), int(i), causal)

    work, merge, refs = desc["work"], desc["merge"], desc["refs"]
    info = desc["info"]
    assert info["num_work"] == len(work) and info["num_merge"] == len(merge)
    assert info["num_merge_refs"] == len(refs)
    T = int(qo[-1])
    row_of_token = np.repeat(np.arange(B), np.diff(qo))
    cover = [[] for _ in range(T)]  # (key_begin, key_end, item index)
    ws_used = []
    n_cascade = 0
    for wi, (q_row0, n_rows, page_base, kv_len, kb, ke, diag, partial) in enumerate(work):
        assert q_row0 % H == 0 and n_rows % H == 0 and 0 < n_rows <= 128
        t0, ntok = q_row0 // H, n_rows // H
        rows = set(row_of_token[t0:t0 + ntok].tolist())
        assert kb % M.MLA_KEY_TILE == 0 and (kb <= ke or (kb == ke))
        if len(rows) > 1 or (kv_len != k_att[row_of_token[t0]]):
            # a cascade item: a shared prefix [0, kv_len) seen in full by every row
            n_cascade += 1
            assert partial >= 0 and kb >= 0 and ke <= kv_len and diag >= kv_len
            # it reads some row's pages (the group's first); every row it serves names
            # the same page ids for those keys
            assert page_base in set(kvp[:-1].tolist())
            npg = -(-int(kv_len) // P)
            for b in rows:
                assert np.array_equal(idx[kvp[b]:kvp[b] + npg], idx[page_base:page_base + npg])
            for tt in range(ntok):
                b = row_of_token[t0 + tt]
                assert kv_len <= vis_of(b, t0 + tt - qo[b])
                assert min(max(diag + tt + 1, 0), kv_len) == kv_len
                cover[t0 + tt].append((kb, ke, wi))
        else:
            b = row_of_token[t0]
            assert page_base == kvp[b]  # so key j -> kv_indices[page_base + j // P], slot j % P
            i0 = t0 - qo[b]
            assert ke <= max(vis_of(b, i0 + ntok - 1), kb)
            for tt in range(ntok):
                # the kernel's rule: keys < clamp(diag + tt + 1, 0, kv_len)
                assert min(max(diag + tt + 1, 0), kv_len) == vis_of(b, i0 + tt)
                cover[t0 + tt].append((kb, ke, wi))
        if partial >= 0:
            ws_used.append((int(partial), int(partial) + int(n_rows)))
    # (a single-row prefix item whose prefix is all of the row reads like an ordinary one)
    assert n_cascade <= info["num_cascade"]
    # partial results occupy disjoint workspace rows
    ws_used.sort()
    for (a0, a1), (b0, b1) in zip(ws_used, ws_used[1:]):
        assert a1 <= b0
    assert info["num_partials"] == len(ws_used)
    # every visible key of every query is covered exactly once
    for t in range(T):
        b = row_of_token[t]
        vis = vis_of(b, t - qo[b])
        spans = sorted((kb, ke) for kb, ke, _ in cover[t])
        assert spans, f"token {t} uncovered"
        pos = 0
        for (kb, ke) in spans:
            if ke <= kb:
                continue
            assert kb == pos, f"token {t}: gap/overlap at {pos} vs {kb}"
            pos = ke
        assert pos >= vis  # keys past a token's own limit are masked by the kernel's rule
    # merges: a token with partial items is combined once, from exactly those partials
    merged_by = [None] * T
    for mi, (q_row0, n_rows, first, n) in enumerate(merge):
        assert n >= 1 and q_row0 % H == 0 and n_rows % H == 0
        for t in range(q_row0 // H, (q_row0 + n_rows) // H):
            assert merged_by[t] is None
            merged_by[t] = mi
        assert 0 <= first and first + n <= len(refs)
    for t in range(T):
        parts = [wi for _, _, wi in cover[t] if work[wi][7] >= 0]
        finals = [wi for _, _, wi in cover[t] if work[wi][7] < 0]
        if not parts:
            assert merged_by[t] is None and len(finals) == 1
            continue
        assert not finals and merged_by[t] is not None
        q_row0, n_rows, first, n = merge[merged_by[t]]
        # the workspace row that holds token t's head 0 in each referenced partial
        want = sorted(int(work[wi][7]) + (t * H - int(work[wi][0])) for wi in parts)
        got = sorted(int(r) + (t * H - int(q_row0)) for r in refs[first:first + n])
        assert got == want
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


def test_small_decode_splits_for_latency_within_one_wave():
    """With fewer items than SM pairs the step lasts as long as its longest item: the
    tiny decode step's 3-tile row is cut into single tiles (4 items, one merge), while a
    step whose single-tile split would exceed one wave keeps its throughput split."""
    d = make_config("tiny_decode", tables_only=True)
    desc = M.mla_plan_describe(plan_tables(d))
    assert desc["info"]["num_work"] == 4 and desc["info"]["num_merge"] == 1
    assert max(w[5] - w[4] for w in desc["work"]) <= M.MLA_KEY_TILE
    check_layout(d, desc)
    d8 = make_custom([1] * 8, [300 + 97 * i for i in range(8)], 128, 64, seed=5, tables_only=True)
    desc = M.mla_plan_describe(plan_tables(d8))
    assert desc["info"]["num_work"] <= 74
    check_layout(d8, desc)


@pytest.mark.parametrize("H,P,q", [(128, 64, 4), (16, 16, 4), (16, 16, 3), (32, 32, 1), (64, 128, 2), (64, 64, 1)])
def test_cascade_layout_covers_once_and_groups_rows(H, P, q):
    """Shared-prefix cascade (consecutive rows naming the same first pages attend them
    together): coverage, visibility and merge references stay exact; a group gets
    prefix tiles exactly where one tile packs the queries of two or more rows."""
    B, group = 12, 4
    k = [1024 + q + 13 * i for i in range(B)]
    d = make_custom([q] * B, k, H, P, shared_group=group, shared_pages=1024 // P, tables_only=True, seed=H + P)
    p = plan_tables(d, cascade=True)
    desc = M.mla_plan_describe(p)
    check_layout(d, desc)
    info = desc["info"]
    per_tile = 128 // (H * q) if H * q <= 128 else 1  # rows' query tiles per prefix tile
    if per_tile < 2:
        assert info["num_cascade"] == 0  # nothing to pack: the plan is the plain one
    else:
        tiles = (B // group) * (-(-group // per_tile))
        prefix = [w for w in desc["work"] if w[6] >= w[3] and w[1] > H * q]
        assert info["num_cascade"] >= tiles and len(prefix) >= tiles
        assert all(w[1] <= 128 for w in prefix)
    # without the option, nothing is cascaded
    assert M.mla_plan_describe(plan_tables(d))["info"]["num_cascade"] == 0


def test_cascade_skips_groups_without_a_full_tile_of_prefix():
    d = make_custom([2] * 8, [700] * 8, 128, 16, shared_group=4, shared_pages=3, tables_only=True)
    desc = M.mla_plan_describe(plan_tables(d, cascade=True))
    check_layout(d, desc)
    assert desc["info"]["num_cascade"] == 0  # 48 shared keys < one 64-key tile


@pytest.mark.parametrize("split", [0, -1, 128])
def test_context_only_layout(split):
    """Context-only plans attend keys [0, k_b - q_b) of every row with no causal mask."""
    rng = np.random.default_rng(7 + split)
    q = rng.integers(1, 40, 10).tolist()
    k = [qi + int(c) for qi, c in zip(q, rng.integers(0, 900, 10))]
    k[2] = q[2]  # no stored context
    d = make_custom(q, k, 64, 32, tables_only=True, seed=3)
    desc = M.mla_plan_describe(plan_tables(d, context_only=True, split_keys=split))
    check_layout(d, desc, context_only=True)
    # a row whose tables lack slots for its own tokens is rejected
    bad = make_custom([5], [3], 64, 32, tables_only=True)
    with pytest.raises(M.MlaError):
        plan_tables(bad, context_only=True)


def test_update_recognises_an_unchanged_step_and_replans_otherwise():
    # one page pool for both steps: a plan's geometry (num_pages) is fixed
    d1 = make_custom([1] * 6, [300, 900, 64, 4000, 17, 2000], 128, 64, tables_only=True, seed=1, pool_pages=400)
    d2 = make_custom([2] * 5, [700, 60, 3000, 128, 9000], 128, 64, tables_only=True, seed=2, pool_pages=400)
    p = plan_tables(d1)
    assert M.mla_plan_update(p, d1.qo_indptr, d1.kv_indptr, d1.kv_indices, d1.last_page_len)
    assert not M.mla_plan_update(p, d2.qo_indptr, d2.kv_indptr, d2.kv_indices, d2.last_page_len)
    check_layout(d2, M.mla_plan_describe(p))
    assert M.mla_plan_update(p, d2.qo_indptr, d2.kv_indptr, d2.kv_indices, d2.last_page_len)
    # one changed page id is a different step
    kvi = d2.kv_indices.clone()
    kvi[3] = (int(kvi[3]) + 1) % d2.num_pages
    assert not M.mla_plan_update(p, d2.qo_indptr, d2.kv_indptr, kvi, d2.last_page_len)


def test_graph_plan_bounds_hold_across_steps():
    """A graph plan's layout fits its bucket's fixed capacity for every step that fits
    the bucket; a step beyond the bucket is rejected and leaves the plan as it was."""
    kw = dict(graph_max_batch=16, graph_max_tokens=64, graph_max_page_ids=2048)
    d0 = make_custom([1] * 16, [100 + 300 * i for i in range(16)], 128, 64, tables_only=True, seed=4,
                     pool_pages=4096)
    p = plan_tables(d0, **kw)
    cap = M.mla_plan_get_info(p)["work_capacity"]
    assert M.mla_plan_get_info(p)["graph"] == 1
    rng = np.random.default_rng(5)
    for step in range(6):
        B = int(rng.integers(1, 17))
        q = rng.integers(1, 5, B).tolist()
        k = [int(qi + x) for qi, x in zip(q, rng.integers(0, 8000, B))]
        d = make_custom(q, k, 128, 64, tables_only=True, seed=10 + step, pool_pages=4096)
        if int(d.kv_indptr[-1]) > 2048 or sum(q) > 64:
            continue
        M.mla_plan_update(p, d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len)
        desc = M.mla_plan_describe(p)
        check_layout(d, desc)
        assert desc["info"]["num_work"] <= cap and desc["info"]["work_capacity"] == cap
    too_many = make_custom([1] * 17, [64] * 17, 128, 64, tables_only=True, pool_pages=4096)
    before = M.mla_plan_describe(p)["work"].copy()
    with pytest.raises(M.MlaError):
        M.mla_plan_update(p, too_many.qo_indptr, too_many.kv_indptr, too_many.kv_indices, too_many.last_page_len)
    assert np.array_equal(M.mla_plan_describe(p)["work"], before)
    # the three bounds go together
    with pytest.raises(M.MlaError):
        plan_tables(d0, graph_max_batch=16, graph_max_tokens=64)


@pytest.mark.parametrize("H,P,q", [(16, 16, 4), (32, 32, 2), (64, 64, 1)])
def test_cascade_with_context_only_layout(H, P, q):
    """Both options together: the shared prefix is cut to the stored context every query
    of the group sees (c_b = k_b - q_b), and coverage stays exact."""
    B, group = 8, 4
    k = [1024 + q + 64 + 29 * i for i in range(B)]
    d = make_custom([q] * B, k, H, P, shared_group=group, shared_pages=1024 // P, tables_only=True, seed=H)
    desc = M.mla_plan_describe(plan_tables(d, cascade=True, context_only=True))
    check_layout(d, desc, context_only=True)
    assert desc["info"]["num_cascade"] > 0


def test_graph_plan_with_cascade_stays_within_capacity():
    kw = dict(graph_max_batch=16, graph_max_tokens=64, graph_max_page_ids=4096, cascade=True)
    d0 = make_custom([4] * 16, [1100 + 50 * i for i in range(16)], 16, 16, shared_group=8, shared_pages=64,
                     tables_only=True, seed=8, pool_pages=6000)
    p = plan_tables(d0, **kw)
    cap = M.mla_plan_get_info(p)["work_capacity"]
    desc = M.mla_plan_describe(p)
    check_layout(d0, desc)
    assert desc["info"]["num_cascade"] > 0 and desc["info"]["num_work"] <= cap
    d1 = make_custom([2] * 12, [2000 + 70 * i for i in range(12)], 16, 16, shared_group=4, shared_pages=100,
                     tables_only=True, seed=9, pool_pages=6000)
    M.mla_plan_update(p, d1.qo_indptr, d1.kv_indptr, d1.kv_indices, d1.last_page_len)
    desc = M.mla_plan_describe(p)
    check_layout(d1, desc)
    assert desc["info"]["num_work"] <= cap


# ----------------------------------------------------------------------------- properties
from hypothesis import HealthCheck, given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@st.composite
def _step(draw):
    H = draw(st.sampled_from([16, 32, 64, 128]))
    P = draw(st.sampled_from([16, 32, 64, 128]))
    B = draw(st.integers(0, 10))
    q = [draw(st.integers(0, 24)) for _ in range(B)]
    k = [draw(st.integers(0, 900)) for _ in range(B)]
    causal = draw(st.booleans())
    context_only = draw(st.booleans())
    if context_only:
        k = [max(ki, qi) for ki, qi in zip(k, q)]
    group = draw(st.sampled_from([0, 2, 3]))
    shared = 0
    if group and B and min(k) >= 2 * P:
        shared = draw(st.integers(1, min(k) // P))
    split = draw(st.sampled_from([0, 0, -1, 64, 192, 512]))
    cascade = draw(st.booleans())
    return dict(H=H, P=P, q=q, k=k, causal=causal, context_only=context_only, group=group, shared=shared,
                split=split, cascade=cascade)


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(_step())
def test_random_steps_keep_exact_bookkeeping(c):
    """Any valid step, with any mix of options, plans to work items that cover every
    visible key of every query exactly once, with merge references that reach every
    partial once and a kernel visibility rule that matches the oracle's."""
    d = make_custom(c["q"], c["k"], c["H"], c["P"], causal=c["causal"], tables_only=True, extra_pool_pages=2,
                    shared_group=c["group"] if c["shared"] else 0, shared_pages=c["shared"])
    p = plan_tables(d, split_keys=c["split"], cascade=c["cascade"], context_only=c["context_only"])
    desc = M.mla_plan_describe(p)
    check_layout(d, desc, context_only=c["context_only"])
    if c["split"] > 0:
        assert all(w[5] - w[4] <= c["split"] for w in desc["work"])


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(st.lists(st.tuples(st.lists(st.integers(0, 6), min_size=1, max_size=8),
                          st.lists(st.integers(0, 3000), min_size=8, max_size=8)), min_size=2, max_size=5),
       st.sampled_from([16, 64, 128]), st.booleans())
def test_graph_plan_sequences_keep_bookkeeping_and_capacity(steps, H, cascade):
    """A graph plan re-planned through a random sequence of steps of its bucket keeps
    exact bookkeeping and never exceeds the launch capacity it was made with; a step
    outside the bucket is rejected without changing the plan."""
    pool = 500
    first = None
    plan = None
    cap = None
    for q, k in steps:
        k = [max(ki, 1) for ki in k[: len(q)]]
        d = make_custom(q, k, H, 64, tables_only=True, pool_pages=pool, seed=len(q) + sum(k) % 97)
        if int(d.kv_indptr[-1]) > 400 or sum(q) > 48:
            continue
        if plan is None:
            plan = plan_tables(d, graph_max_batch=8, graph_max_tokens=48, graph_max_page_ids=400, cascade=cascade)
            cap = M.mla_plan_get_info(plan)["work_capacity"]
            first = d
        else:
            M.mla_plan_update(plan, d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len)
        desc = M.mla_plan_describe(plan)
        check_layout(d, desc)
        assert desc["info"]["num_work"] <= cap and desc["info"]["work_capacity"] == cap
    if plan is not None:
        before = M.mla_plan_describe(plan)["work"].copy()
        big = make_custom([1] * 9, [64] * 9, H, 64, tables_only=True, pool_pages=pool)  # 9 rows > 8
        with pytest.raises(M.MlaError):
            M.mla_plan_update(plan, big.qo_indptr, big.kv_indptr, big.kv_indices, big.last_page_len)
        assert np.array_equal(M.mla_plan_describe(plan)["work"], before)
        assert first is not None
