"""GPU parity: the sm_100a library (through its C ABI) against the fp64 oracle.

Tolerances (fixed by the latent-attention target): bf16 output
|err| <= 1e-2 + 1e-2 * |ref|; lse |err| <= 1e-3 (and -inf exactly where the oracle
has -inf).  Small cases compare every element.  The four full-size workloads are planned as the
benchmark plans them; every token of decode_b64, long_decode and spec_shared_prefix is
compared, and on mixed_prefill every decode row, every merged tile and one token in
eight (plus the first and last) of each 1024-token prefill row.
"""

import numpy as np
import pytest
import torch

import paged_head_latent_mla_b200 as M
from oracle import mla_oracle as O
from workloads import CONFIG_NAMES, make_config, make_custom

pytestmark = pytest.mark.gpu

OUT_ATOL, OUT_RTOL, LSE_ATOL = 1e-2, 1e-2, 1e-3
TEST_TIMEOUT_NS = 500_000_000  # a broken wait fails the test in 0.5 s instead of 4 s


@pytest.fixture(scope="module", autouse=True)
def lib():
    from paged_head_latent_mla_b200 import _build

    _build.build()
    return M.load_library()


def gpu_run(d, split_keys=0, return_lse=True, timeout_ns=TEST_TIMEOUT_NS, plan_kw=None):
    dev = torch.device("cuda:0")
    plan = M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=d.num_heads,
                      page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, causal=d.causal,
                      split_keys=split_keys, wait_timeout_ns=timeout_ns, **(plan_kw or {}))
    qn, qp, cache = d.q_nope.to(dev), d.q_pe.to(dev), d.cache.to(dev)
    res = M.mla_run(plan, qn, qp, cache, return_lse=return_lse)
    status = M.mla_plan_check(plan)
    assert status == M.MLA_OK, M.status_string(status)
    out, lse = res if return_lse else (res, None)
    info = M.mla_plan_get_info(plan)
    desc = M.mla_plan_describe(plan)
    plan.destroy()
    return out.float().cpu().numpy(), (lse.cpu().numpy() if lse is not None else None), info, desc


def compare(d, out, lse, tokens=None):
    ref_o, ref_l = O.mla_attention(d.q_nope, d.q_pe, d.cache, d.qo_indptr, d.kv_indptr, d.kv_indices,
                                   d.last_page_len, d.page_size, d.sm_scale, causal=d.causal, tokens=tokens)
    sel = slice(None) if tokens is None else np.asarray(sorted(set(int(t) for t in tokens)))
    ro, go = ref_o[sel], out[sel]
    err = np.abs(go - ro)
    bound = OUT_ATOL + OUT_RTOL * np.abs(ro)
    bad = err > bound
    assert not bad.any(), (f"out mismatch at {np.argwhere(bad)[:5].tolist()}: max err {err.max():.3e}, "
                           f"gpu {go[bad][:5]}, ref {ro[bad][:5]}")
    if lse is not None:
        rl, gl = ref_l[sel], lse[sel]
        inf_r = np.isneginf(rl)
        assert np.array_equal(inf_r, np.isneginf(gl)), "lse -inf pattern differs"
        if (~inf_r).any():
            le = np.abs(gl[~inf_r] - rl[~inf_r])
            assert le.max() <= LSE_ATOL, f"lse max err {le.max():.3e}"
    return float(err.max()) if err.size else 0.0


# ----------------------------------------------------------------------------- small cases
def test_tiny_decode_config():
    d = make_config("tiny_decode")
    out, lse, info, _ = gpu_run(d)
    # the 3-tile row is cut into single tiles for latency (4 items, one merge)
    assert info["num_work"] == 4 and info["num_merge"] == 1
    compare(d, out, lse)
    out1, lse1, info1, _ = gpu_run(d, split_keys=-1)  # and unsplit
    assert info1["num_work"] == 2
    compare(d, out1, lse1)


@pytest.mark.parametrize("H", [16, 32, 64, 128])
@pytest.mark.parametrize("P", [16, 32, 64, 128])
def test_heads_and_page_sizes(H, P):
    rng = np.random.default_rng(H * 7 + P)
    q = [1, 3, 9, 1, 17]
    k = [int(x) for x in rng.integers(1, 400, len(q))]
    k[2] = 200  # prefill-ish row
    d = make_custom(q, k, H, P, seed=H + P, extra_pool_pages=5)
    out, lse, _, _ = gpu_run(d)
    compare(d, out, lse)


@pytest.mark.parametrize("causal", [True, False])
def test_multi_tile_ragged(causal):
    # several 64-key tiles, ragged tails, queries spanning several 128-row tiles (H=16)
    d = make_custom([1, 20, 33, 7], [65, 191, 300, 64], 16, 16, causal=causal, seed=3)
    out, lse, _, _ = gpu_run(d)
    compare(d, out, lse)


def test_empty_rows_and_overhang():
    # k = 0 with queries; q > k (causal: first queries see nothing); a zero-query row
    d = make_custom([3, 6, 0, 2], [0, 4, 50, 130], 32, 16, causal=True, seed=5)
    out, lse, _, _ = gpu_run(d)
    compare(d, out, lse)
    assert np.all(out[0:3] == 0) and np.all(np.isneginf(lse[0:3]))
    assert np.all(out[3:5] == 0) and np.all(np.isneginf(lse[3:5]))


@pytest.mark.parametrize("split", [64, 128, 320])
def test_forced_split_matches_oracle(split):
    d = make_custom([1, 1, 5, 2], [1000, 64, 777, 1500], 64, 64, seed=11)
    out, lse, info, _ = gpu_run(d, split_keys=split)
    assert info["num_merge"] > 0
    compare(d, out, lse)


def test_split_without_lse_output():
    d = make_custom([1, 2], [900, 1300], 128, 64, seed=12)
    out, lse, info, _ = gpu_run(d, split_keys=128, return_lse=False)
    assert info["num_merge"] > 0 and lse is None
    compare(d, out, None)


def test_shared_prefix_small():
    q = [4] * 16
    k = [1024 + 97 * i for i in range(16)]
    d = make_custom(q, k, 128, 64, shared_group=8, shared_pages=16, seed=13)
    out, lse, _, _ = gpu_run(d)
    compare(d, out, lse)


def test_single_visible_key_is_exact():
    # k = 1 rows, and the first query of a causal row with q == k: weight exactly 1
    d = make_custom([1, 4], [1, 4], 64, 16, seed=17)
    out, lse, _, _ = gpu_run(d)
    cache = d.cache.float().numpy()
    idx = d.kv_indices.numpy()
    kvp = d.kv_indptr.numpy()
    for t, b in [(0, 0), (1, 1)]:
        key = cache[idx[kvp[b]], 0, :512]
        assert np.array_equal(out[t], np.broadcast_to(key, out[t].shape))
    compare(d, out, lse)


def test_page_permutation_bit_identical():
    d = make_custom([1, 3, 2], [300, 129, 64], 32, 16, seed=19, extra_pool_pages=7)
    out1, lse1, _, _ = gpu_run(d)
    g = torch.Generator().manual_seed(1)
    perm = torch.randperm(d.num_pages, generator=g)
    cache2 = torch.empty_like(d.cache)
    cache2[perm] = d.cache
    d2 = make_custom([1, 3, 2], [300, 129, 64], 32, 16, seed=19, extra_pool_pages=7)
    d2.cache = cache2
    d2.kv_indices = perm[d.kv_indices.long()].to(torch.int32)
    out2, lse2, _, _ = gpu_run(d2)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


def test_causal_is_noop_for_single_query():
    d = make_custom([1, 1, 1], [77, 500, 1], 128, 32, seed=23)
    a = gpu_run(d)
    d.causal = False
    b = gpu_run(d)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_repeat_runs_deterministic():
    d = make_custom([1, 5], [700, 900], 128, 64, seed=29)
    a = gpu_run(d, split_keys=256)
    b = gpu_run(d, split_keys=256)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ----------------------------------------------------------------------------- full sizes
def _full_size_tokens(d, desc, stride=8, seed=0):
    """Tokens of a full-size workload the oracle checks one by one.

    Every token of every row with at most ``stride`` queries (all of decode_b64,
    long_decode and spec_shared_prefix, and the decode rows of mixed_prefill); for
    longer rows the first and last token and one token in every ``stride`` (a seeded
    phase per row); and every token of every query tile the merge kernel combines
    (split or cascaded tiles)."""
    qo = d.qo_indptr.numpy()
    H = d.num_heads
    rng = np.random.default_rng(seed)
    toks = set()
    for b in range(len(qo) - 1):
        t0, t1 = int(qo[b]), int(qo[b + 1])
        if t1 == t0:
            continue
        if t1 - t0 <= stride:
            toks.update(range(t0, t1))
            continue
        toks.update({t0, t1 - 1})
        toks.update(range(t0 + int(rng.integers(0, stride)), t1, stride))
    for (q_row0, n_rows, _first, _n) in desc["merge"]:
        toks.update(range(int(q_row0) // H, (int(q_row0) + int(n_rows) - 1) // H + 1))
    return sorted(toks)


@pytest.mark.slow
@pytest.mark.parametrize("name", [n for n in CONFIG_NAMES if n != "tiny_decode"])
def test_full_size_config_against_oracle(name):
    """The four full-size workloads, planned as the benchmark plans them (automatic split),
    run once with the benchmark's lse setting and once with lse on; the output is checked
    element by element on every token of every short row, on every token of every merged
    tile and on one token in eight (plus the first and last) of each long prefill row."""
    d = make_config(name)
    out, lse, info, desc = gpu_run(d, return_lse=True)
    toks = _full_size_tokens(d, desc)
    compare(d, out, lse, tokens=toks)
    # properties that hold at any size: every query sees >= 1 key here, so every output
    # is finite and every lse finite
    assert np.isfinite(out).all() and np.isfinite(lse).all()
    if not d.return_lse:
        out2, _, _, _ = gpu_run(d, return_lse=False)  # the benchmark's launch (no lse)
        assert np.array_equal(out, out2)
    if name in ("decode_b64", "long_decode", "spec_shared_prefix"):
        assert len(toks) == d.total_tokens  # every token was compared


def test_page_named_twice_within_a_row():
    """A row whose page list names the same physical page twice (pure indexing: the keys
    at both positions are that page's rows), next to rows that share its pages."""
    d = make_custom([1, 3, 2], [700, 520, 300], 128, 64, seed=31, extra_pool_pages=4)
    idx = d.kv_indices.clone()
    kvp = d.kv_indptr.numpy()
    idx[kvp[0] + 5] = idx[kvp[0] + 1]   # row 0: page list position 5 repeats position 1
    idx[kvp[0] + 8] = idx[kvp[0] + 1]   # ... and position 8 (its last page, partly used)
    idx[kvp[1] + 2] = idx[kvp[1] + 0]   # row 1 repeats its first page
    idx[kvp[2] + 1] = idx[kvp[0] + 3]   # row 2 names a page of row 0
    d.kv_indices = idx
    out, lse, _, _ = gpu_run(d)
    compare(d, out, lse)
    out2, lse2, _, _ = gpu_run(d, split_keys=128)  # and through split partials
    compare(d, out2, lse2)


def test_pooled_plan_buffers_reused_across_shapes():
    """mla_plan takes its device blob, split-KV workspace and pinned staging from a pool
    that mla_plan_destroy refills.  Alternate plans of different sizes (so a plan often
    receives a buffer that still holds another plan's work list or partials), keep two
    plans alive at once (they must not share a buffer), and check every result."""
    dev = torch.device("cuda:0")
    cases = [make_custom([1, 1, 2], [9000, 300, 4100], 128, 64, seed=61),       # split partials
             make_custom([3, 0, 1], [40, 7, 1300], 32, 16, seed=62),            # small, unsplit
             make_custom([1] * 6, [5000 + 700 * i for i in range(6)], 64, 32, seed=63)]

    def plan_of(d, split):
        return M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=d.num_heads,
                          page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, causal=d.causal,
                          split_keys=split, wait_timeout_ns=TEST_TIMEOUT_NS)

    refs = [O.mla_attention(d.q_nope, d.q_pe, d.cache, d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len,
                            d.page_size, d.sm_scale, causal=d.causal) for d in cases]
    inputs = [(d.q_nope.to(dev), d.q_pe.to(dev), d.cache.to(dev)) for d in cases]

    def check(i, out, lse):
        ro, rl = refs[i]
        o = out.float().cpu().numpy()
        assert (np.abs(o - ro) <= OUT_ATOL + OUT_RTOL * np.abs(ro)).all()
        gl = lse.cpu().numpy()
        inf = np.isneginf(rl)
        assert np.array_equal(inf, np.isneginf(gl))
        if (~inf).any():
            assert np.abs(gl[~inf] - rl[~inf]).max() <= LSE_ATOL

    for rnd, order in enumerate(([0, 1, 2], [2, 0, 1], [1, 2, 0])):
        for i in order:
            plan = plan_of(cases[i], 128 if rnd % 2 == 0 else 0)
            out, lse = M.mla_run(plan, *inputs[i], return_lse=True)
            assert M.mla_plan_check(plan) == M.MLA_OK
            plan.destroy()
            check(i, out, lse)
    # two live plans at once
    a, b = plan_of(cases[0], 192), plan_of(cases[2], 128)
    oa, la = M.mla_run(a, *inputs[0], return_lse=True)
    ob, lb = M.mla_run(b, *inputs[2], return_lse=True)
    assert M.mla_plan_check(a) == M.MLA_OK and M.mla_plan_check(b) == M.MLA_OK
    check(0, oa, la)
    check(2, ob, lb)
    a.destroy()
    b.destroy()


def _with_common_offset(d, q_shift, k_shift, seed):
    """The same step with a shared direction added to every query and every key: each
    score gains about q_shift * k_shift * 576 * sm_scale, the same for every key of a
    row up to the keys' own spread, so the scores sit far from zero while their
    differences stay those of the random parts."""
    g = torch.Generator().manual_seed(seed)
    u = torch.randn(576, generator=g)
    u = u / u.norm()
    d.q_nope = (d.q_nope.float() + q_shift * u[:512]).to(torch.bfloat16)
    d.q_pe = (d.q_pe.float() + q_shift * u[512:]).to(torch.bfloat16)
    d.cache = (d.cache.float() + k_shift * u).to(torch.bfloat16)
    return d


def test_scores_far_from_zero():
    """Scores near +300 natural units, with the usual spread between keys.  The pair of
    CTAs exchanges its partial scores as 16-bit offsets below a per-row anchor, so the
    precision must not depend on the scores' distance from zero."""
    d = make_custom([1, 4, 1], [900, 300, 2000], 128, 64, seed=37)
    d = _with_common_offset(d, 60.0, 60.0, seed=38)  # 60 * 60 * 0.072 = 260 in the score
    out, lse, _, _ = gpu_run(d)
    compare(d, out, lse)
    assert np.nanmin(lse) > 200  # the offset is really there


def test_opposite_half_partials():
    """Keys whose large scores come from opposite halves of the latent width: key A's
    from ckv columns [0, 256) and kpe [0, 32), key B's from ckv [256, 512) and kpe
    [32, 64), the two halves that the two CTAs of a pair hold.  Each CTA then sees one
    key's partial far above the other's (about 150 natural units apart), while their
    full scores are equal.  The partials travel between the CTAs in a 16-bit code
    whose step follows each row's span, so both keys keep equal weight, as the oracle
    has them, alongside keys with a wide random spread of scores from the rope part."""
    d = make_custom([1, 1, 3], [40, 100, 130], 16, 16, seed=41)
    g = torch.Generator().manual_seed(42)
    c = d.cache.float()
    c[..., 512:] *= torch.exp(torch.randn((d.num_pages, d.page_size, 1), generator=g) * 1.5) * 4.0
    qn, qp = d.q_nope.float(), d.q_pe.float()
    qv = torch.cat([qn[0, 0], qp[0, 0]])  # row 0's query (all its heads share it)
    qn[0, :] = qv[:512]
    qp[0, :] = qv[512:]
    half0 = torch.zeros(576, dtype=torch.bool)
    half0[:256] = True
    half0[512:544] = True
    target = 150.0 / d.sm_scale  # score of 150 natural units
    kvp, idx = d.kv_indptr.numpy(), d.kv_indices.numpy()
    for key, mask in ((5, half0), (27, ~half0)):
        page, slot = int(idx[kvp[0] + key // d.page_size]), key % d.page_size
        v = torch.where(mask, qv, torch.zeros_like(qv))
        c[page, slot] = v * (target / float(v @ v))
    d.cache, d.q_nope, d.q_pe = c.to(torch.bfloat16), qn.to(torch.bfloat16), qp.to(torch.bfloat16)
    out, lse, _, _ = gpu_run(d)
    compare(d, out, lse)


@pytest.mark.parametrize("kv", [[2100, 300], [4500, 64]])
def test_merge_of_many_partials(kv):
    """Split tiles with more than 32 partials (33 and 71 chunks of 64 keys): the merge
    takes them 32 at a time against a running maximum of their log-sum-exps."""
    d = make_custom([2, 1], kv, 64, 64, seed=13)
    out, lse, info, _ = gpu_run(d, split_keys=64)
    assert info["num_merge_refs"] > 32
    compare(d, out, lse)


def test_very_long_row():
    """One decode token over 262,144 keys (4096 pages, 302 MB of cache) next to a short
    row: the planner spreads the long row over many work items, so its query tile is
    merged from more than 32 partials (the merge's running-maximum path at scale), and
    page and key indices reach their largest values in the suite.  Compared in full."""
    d = make_custom([1, 1], [262_144, 300], 128, 64, seed=31)
    out, lse, info, _ = gpu_run(d)
    assert info["num_merge"] >= 1 and info["num_merge_refs"] > 32
    compare(d, out, lse)


def test_large_batch_of_short_rows():
    """2048 decode rows of 1 to 600 keys in 16-key pages (two TMA boxes per key tile;
    many rows shorter than one tile; at 64 heads a query tile holds two tokens, but a
    tile never spans rows, so each row has its own): thousands of work items through
    the planner and the kernel; every 8th row and the last are compared with the oracle."""
    g = np.random.default_rng(37)
    kv = [int(x) for x in g.integers(1, 601, size=2048)]
    d = make_custom([1] * 2048, kv, 64, 16, seed=37)
    out, lse, info, _ = gpu_run(d)
    assert info["num_work"] >= 2048
    compare(d, out, lse, tokens=list(range(0, 2048, 8)) + [2047])


def test_long_causal_prefill_small_heads():
    """A 1000-token causal prefill over 3000 keys at 16 heads (8 tokens per query tile, so
    the causal edge runs through every tile) in 128-key pages, beside a decode row:
    every 7th token, the first and last of the row, and the tokens around tile edges are
    compared with the oracle."""
    d = make_custom([1000, 1], [3000, 2222], 16, 128, seed=41)
    out, lse, _, _ = gpu_run(d)
    toks = set(range(0, 1000, 7)) | {0, 999, 1000} | {t for b in range(8, 1000, 128) for t in (b - 1, b)}
    compare(d, out, lse, tokens=sorted(toks))
