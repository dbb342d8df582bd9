"""Pins for the fp64 oracle: each check ties it to something other than itself.

* explicit 192-wide per-head attention with generated W_UK / W_UV (the absorbed
  form of the flashinfer_mla page's module description must equal it);
* torch's own scaled_dot_product_attention with a lower-right causal bias (a
  library routine for end-aligned causal attention, ragged.wrappers page,
  PrefixedPrefillWrapper);
* a hand-derived worked example stored under tests/golden/;
* closed forms (zero query, equal keys, a single visible key);
* invariances (physical page permutation; causal == non-causal for one query);
* the LSE merge identity (flashinfer_mla page, FlashInferMLAManager.run: the lse
  exists to merge key segments), with brute-force splits;
* the cache append against a walk over the page lists and a hand-derived example,
  and its round trip through the paged gather;
* context-only attention merged with attention over the step's own tokens equals
  full causal attention (the two key sets partition every query's visible keys).

The ``check_*`` functions take the oracle module as an argument so that the
mutation tests at the bottom can plant plausible mistakes in a copy of the
oracle (on the CPU) and show that some pin catches each one.
"""

import importlib.util
import json
import math
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")

from oracle import mla_oracle as O  # noqa: E402

D_C, D_R = 512, 64
SCALE = 192 ** -0.5


def _paged(q_lens, kv_lens, H, page_size, seed, std=0.5, pool_extra=3, shuffle=True):
    """Small fp64 paged inputs built directly here (values need not be bf16 for the
    oracle); returns a dict of numpy arrays."""
    rng = np.random.default_rng(seed)
    n_pages = [-(-k // page_size) for k in kv_lens]
    pool = sum(n_pages) + pool_extra
    perm = rng.permutation(pool) if shuffle else np.arange(pool)
    indices, kvp, cur = [], [0], 0
    for n in n_pages:
        indices.extend(perm[cur : cur + n].tolist())
        cur += n
        kvp.append(kvp[-1] + n)
    last = [k - (n - 1) * page_size if n else 1 for k, n in zip(kv_lens, n_pages)]
    qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int64)
    T = int(qo[-1])
    return dict(
        q_nope=rng.normal(0, std, (T, H, D_C)),
        q_pe=rng.normal(0, std, (T, H, D_R)),
        cache=rng.normal(0, std, (pool, page_size, D_C + D_R)),
        qo_indptr=qo,
        kv_indptr=np.array(kvp, dtype=np.int64),
        kv_indices=np.array(indices, dtype=np.int64),
        last_page_len=np.array(last, dtype=np.int64),
        page_size=page_size,
    )


def _run(oracle, d, causal=True, scale=SCALE):
    return oracle.mla_attention(
        d["q_nope"], d["q_pe"], d["cache"], d["qo_indptr"], d["kv_indptr"], d["kv_indices"],
        d["last_page_len"], d["page_size"], scale, causal=causal)


# --------------------------------------------------------------------------- checks
def check_absorbed_equals_explicit(oracle):
    """Absorbed latent attention == explicit per-head attention with head dim 192
    (128 'nope' + 64 rope) after applying W_UV, on tiny inputs."""
    rng = np.random.default_rng(7)
    H, dn = 3, 128
    q_lens, kv_lens, P = [1, 3, 2], [5, 7, 9], 4
    d = _paged(q_lens, kv_lens, H, P, seed=11)
    W_UK = rng.normal(0, 0.05, (H, dn, D_C))
    W_UV = rng.normal(0, 0.05, (H, dn, D_C))
    T = sum(q_lens)
    q_orig = rng.normal(0, 1.0, (T, H, dn))
    d["q_nope"] = np.einsum("thd,hdc->thc", q_orig, W_UK)  # q_nope @ W_UK, absorbed
    out_lat, lse = _run(oracle, d, causal=True)
    # explicit attention, written independently: per row, keys at absolute positions
    # 0..k-1 and queries at positions k-q..k-1; a query sees keys at or before it.
    t = 0
    for b, (q_b, k_b) in enumerate(zip(q_lens, kv_lens)):
        pages = d["kv_indices"][d["kv_indptr"][b] : d["kv_indptr"][b + 1]]
        lat = [d["cache"][pages[j // P], j % P] for j in range(k_b)]
        for i in range(q_b):
            pos = k_b - q_b + i
            for h in range(H):
                qv = np.concatenate([q_orig[t, h], d["q_pe"][t, h]])
                ks = [np.concatenate([W_UK[h] @ x[:D_C], x[D_C:]]) for x in lat[: pos + 1]]
                vs = [W_UV[h] @ x[:D_C] for x in lat[: pos + 1]]
                sc = [float(qv @ k) * (192 ** -0.5) for k in ks]
                mx = max(sc)
                ws = [math.exp(s - mx) for s in sc]
                z = math.fsum(ws)
                o_exp = sum(w * v for w, v in zip(ws, vs)) / z
                lse_exp = mx + math.log(z)
                np.testing.assert_allclose(W_UV[h] @ out_lat[t, h], o_exp, rtol=1e-10, atol=1e-12)
                assert abs(lse[t, h] - lse_exp) < 1e-10
            t += 1


def check_against_sdpa(oracle):
    """torch SDPA (fp64, CPU) with causal_lower_right == oracle, one row at a time,
    several heads, keys [ckv|kpe] (576), values ckv (512)."""
    from torch.nn.attention.bias import causal_lower_right

    for (q_b, k_b, P, causal) in [(5, 13, 4, True), (1, 9, 8, True), (4, 4, 2, True), (3, 10, 16, False),
                                  (6, 6, 1, True)]:
        H = 2
        d = _paged([q_b], [k_b], H, P, seed=q_b * 100 + k_b)
        out, lse = _run(oracle, d, causal=causal)
        pages = d["kv_indices"]
        K = torch.tensor(np.stack([d["cache"][pages[j // P], j % P] for j in range(k_b)]))
        q = torch.tensor(np.concatenate([d["q_nope"], d["q_pe"]], -1)).permute(1, 0, 2)[None]  # [1,H,q,576]
        k = K[None, None].expand(1, H, k_b, D_C + D_R)
        v = K[None, None, :, :D_C].expand(1, H, k_b, D_C)
        mask = causal_lower_right(q_b, k_b) if causal else None
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=SCALE)
        np.testing.assert_allclose(out, ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)
        sc = (q @ k.transpose(-1, -2)) * SCALE
        if causal:
            sc = sc.masked_fill(~causal_lower_right(q_b, k_b)._materialize(), float("-inf"))
        ref_lse = torch.logsumexp(sc, dim=-1)[0].T.numpy()
        np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-13)


def check_golden_worked_example(oracle):
    with open(os.path.join(GOLDEN, "hand_worked_example.json")) as f:
        g = json.load(f)
    P = g["page_size"]
    cache = np.zeros((g["num_pages"], P, D_C + D_R))
    for (page, slot, col, val) in g["cache_entries"]:
        cache[page, slot, col] = val
    q_nope = np.zeros((1, 1, D_C))
    q_pe = np.zeros((1, 1, D_R))
    for (col, val) in g["q_nope_entries"]:
        q_nope[0, 0, col] = val
    for (col, val) in g["q_pe_entries"]:
        q_pe[0, 0, col] = val
    out, lse = oracle.mla_attention(q_nope, q_pe, cache, np.array([0, 1]), np.array(g["kv_indptr"]),
                                    np.array(g["kv_indices"]), np.array(g["last_page_len"]), P,
                                    g["sm_scale"], causal=True)
    exp = np.zeros(D_C)
    for (col, val) in g["expected_out_entries"]:
        exp[col] = val
    np.testing.assert_allclose(out[0, 0], exp, rtol=0, atol=1e-12)
    assert abs(lse[0, 0] - g["expected_lse"]) < 1e-12


def check_closed_forms(oracle):
    d = _paged([3], [11], 2, 4, seed=5)
    # zero query: every visible key weighs the same -> mean of visible ckv rows, lse = ln(vis)
    d["q_nope"][:] = 0
    d["q_pe"][:] = 0
    out, lse = _run(oracle, d, causal=True)
    pages = d["kv_indices"]
    rows = np.stack([d["cache"][pages[j // 4], j % 4] for j in range(11)])
    for i in range(3):
        vis = 11 - 3 + i + 1
        np.testing.assert_allclose(out[i, 0], rows[:vis, :D_C].mean(0), rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse[i], math.log(vis), rtol=1e-14)
    # all keys equal -> out is that ckv row
    d = _paged([2], [9], 2, 4, seed=6)
    d["cache"][:] = d["cache"][0, 0]
    out, _ = _run(oracle, d, causal=True)
    np.testing.assert_allclose(out, np.broadcast_to(d["cache"][0, 0, :D_C], out.shape), rtol=1e-13)


def check_single_visible_key(oracle):
    # a row with one key, and the first query of a causal row with q_b == k_b
    for q_b, k_b in [(1, 1), (4, 4)]:
        d = _paged([q_b], [k_b], 3, 2, seed=q_b)
        out, lse = _run(oracle, d, causal=True)
        key = d["cache"][d["kv_indices"][0], 0]
        assert np.array_equal(out[0], np.broadcast_to(key[:D_C], (3, D_C)))
        qf = np.concatenate([d["q_nope"][0], d["q_pe"][0]], -1)
        s = np.array([math.fsum(qf[h] * key) for h in range(3)]) * SCALE
        np.testing.assert_allclose(lse[0], s, rtol=1e-12, atol=1e-13)


def check_page_permutation(oracle):
    d = _paged([2, 1, 3], [17, 33, 8], 2, 4, seed=9, pool_extra=5)
    out, lse = _run(oracle, d)
    rng = np.random.default_rng(1)
    pool = d["cache"].shape[0]
    perm = rng.permutation(pool)  # new physical location of each old page
    cache2 = np.empty_like(d["cache"])
    cache2[perm] = d["cache"]
    d2 = dict(d, cache=cache2, kv_indices=perm[d["kv_indices"]])
    out2, lse2 = _run(oracle, d2)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def check_causal_noop_single_query(oracle):
    d = _paged([1, 1, 1], [5, 12, 1], 2, 4, seed=3)
    a = _run(oracle, d, causal=True)
    b = _run(oracle, d, causal=False)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def check_lse_merge(oracle):
    """Attending over keys [0, m) and [m, k) separately and merging by LSE equals
    attending over [0, k), for every split point of a small row (page size 1 makes
    any split expressible as two page lists over the same cache)."""
    k, H = 12, 2
    d = _paged([1], [k], H, 1, seed=21, pool_extra=0)
    full_out, full_lse = _run(oracle, d, causal=False)
    for m in range(0, k + 1):
        pages = d["kv_indices"]
        seg = dict(d, qo_indptr=np.array([0, 1, 2]), kv_indptr=np.array([0, m, k]),
                   kv_indices=pages, last_page_len=np.array([1, 1]),
                   q_nope=np.concatenate([d["q_nope"]] * 2), q_pe=np.concatenate([d["q_pe"]] * 2))
        o, l = _run(oracle, seg, causal=False)
        mo, ml = oracle.merge_states(o[0], l[0], o[1], l[1])
        np.testing.assert_allclose(mo, full_out[0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(ml, full_lse[0], rtol=1e-12, atol=1e-13)
        # three-way merge too
        mo3, ml3 = oracle.merge_many([o[0], o[1], np.zeros_like(o[0])], [l[0], l[1], np.full_like(l[0], -np.inf)])
        np.testing.assert_allclose(mo3, full_out[0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(ml3, full_lse[0], rtol=1e-12, atol=1e-13)


def check_merge_closed_forms(oracle):
    """Closed forms of the two-state merge: an empty state (lse = -inf) is the identity;
    a state merged with itself keeps its output and gains ln 2; two equal-lse states
    average their outputs; a state whose lse is far below the other's leaves it unchanged
    to rounding."""
    rng = np.random.default_rng(41)
    o = rng.normal(size=(5, D_C))
    l = rng.normal(size=5) * 3
    e_o, e_l = np.zeros_like(o), np.full(5, -np.inf)
    mo, ml = oracle.merge_states(o, l, e_o, e_l)
    assert np.array_equal(mo, o) and np.array_equal(ml, l)
    mo, ml = oracle.merge_states(e_o, e_l, e_o, e_l)
    assert np.all(mo == 0) and np.all(np.isneginf(ml))
    mo, ml = oracle.merge_states(o, l, o, l)
    np.testing.assert_allclose(mo, o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(ml, l + math.log(2.0), rtol=0, atol=1e-14)
    o2 = rng.normal(size=(5, D_C))
    mo, ml = oracle.merge_states(o, l, o2, l)
    np.testing.assert_allclose(mo, (o + o2) / 2, rtol=0, atol=1e-14)
    mo, ml = oracle.merge_states(o, l, o2, l - 800.0)
    np.testing.assert_allclose(mo, o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(ml, l, rtol=0, atol=1e-14)


def check_empty_and_overhang(oracle):
    # k = 0 row, and a causal row with more queries than keys
    d = _paged([2, 5], [0, 3], 2, 4, seed=4)
    out, lse = _run(oracle, d, causal=True)
    assert np.all(out[0:2] == 0) and np.all(np.isneginf(lse[0:2]))
    # row 1: q=5, k=3 -> queries 0,1 see nothing; query 2 sees key 0 only
    assert np.all(out[2:4] == 0) and np.all(np.isneginf(lse[2:4]))
    key0 = d["cache"][d["kv_indices"][0], 0]
    assert np.array_equal(out[4], np.broadcast_to(key0[:D_C], (2, D_C)))
    assert np.all(np.isfinite(lse[4:]))


def check_kv_lengths(oracle):
    # brute force: count slots by walking page lists
    kv_indptr = np.array([0, 3, 3, 13, 14])
    last = np.array([5, 1, 6, 16])
    P = 16
    got = oracle.kv_lengths(kv_indptr, last, P)
    want = []
    for b in range(4):
        n = kv_indptr[b + 1] - kv_indptr[b]
        cnt = 0
        for p in range(n):
            cnt += last[b] if p == n - 1 else P
        want.append(cnt)
    assert list(got) == want == [37, 0, 150, 16]
    # page/slot mapping agrees with a walk over the page list
    idx = np.arange(100, 114)
    for b in range(4):
        j = 0
        for p in range(kv_indptr[b], kv_indptr[b + 1]):
            for s in range(last[b] if p == kv_indptr[b + 1] - 1 else P):
                assert oracle.key_location(kv_indptr, idx, P, b, j) == (idx[p], s)
                j += 1


def _walk_slots(kv_indptr, kv_indices, last, P, b):
    """The row's (page, slot) pairs in logical key order, by walking its page list."""
    out = []
    n = kv_indptr[b + 1] - kv_indptr[b]
    for p in range(n):
        for s_ in range(last[b] if p == n - 1 else P):
            out.append((int(kv_indices[kv_indptr[b] + p]), s_))
    return out


def check_append_slots(oracle):
    # hand-derived example
    with open(os.path.join(GOLDEN, "append_tiny.json")) as f:
        g = json.load(f)
    P = g["page_size"]
    cache = np.zeros((g["num_pages"], P, D_C + D_R))
    T = g["qo_indptr"][-1]
    new = np.arange(T, dtype=np.float64)[:, None] + 1.0 + np.zeros((T, D_C + D_R))
    out = oracle.append_latent(cache, new, g["qo_indptr"], g["kv_indptr"], g["kv_indices"], g["last_page_len"], P)
    for t, (page, slot) in enumerate(g["expected_page_slot"]):
        assert np.all(out[page, slot] == t + 1.0)
    assert np.count_nonzero(out.any(axis=-1)) == T  # nothing else written
    # random tables: the last q_b slots of each row's walk receive the new rows in
    # order, every other slot is unchanged, and the paged gather reads them back
    d = _paged([3, 0, 5, 1], [40, 7, 70, 1], 2, 16, seed=11)
    new = np.random.default_rng(12).normal(size=(9, D_C + D_R))
    out = oracle.append_latent(d["cache"], new, d["qo_indptr"], d["kv_indptr"], d["kv_indices"],
                               d["last_page_len"], 16)
    touched = np.zeros(d["cache"].shape[:2], dtype=bool)
    qo = d["qo_indptr"]
    for b in range(4):
        slots = _walk_slots(d["kv_indptr"], d["kv_indices"], d["last_page_len"], 16, b)
        q_b = qo[b + 1] - qo[b]
        for i, (page, slot) in enumerate(slots[len(slots) - q_b:]):
            assert np.array_equal(out[page, slot], new[qo[b] + i])
            touched[page, slot] = True
        k_b = len(slots)
        keys = oracle.gather_row_keys(out, d["kv_indptr"], d["kv_indices"], 16, b, k_b)
        assert np.array_equal(keys[k_b - q_b:], new[qo[b]:qo[b + 1]])
    assert np.array_equal(out[~touched], d["cache"][~touched])
    with pytest.raises(ValueError):
        oracle.append_latent(d["cache"], new[:6], [0, 6], [0, 1], [0], [5], 16)


def check_context_only_merge(oracle):
    """Context-only attention (keys j < k_b - q_b) merged by LSE with attention over the
    row's own q_b tokens (causal among themselves) equals full causal attention."""
    P, H = 16, 3
    q_lens, k_lens = [4, 1, 7, 2], [4 + 37, 1 + 16, 7 + 0, 2 + 50]
    d = _paged(q_lens, k_lens, H, P, seed=21)
    full_o, full_l = oracle.mla_attention(d["q_nope"], d["q_pe"], d["cache"], d["qo_indptr"], d["kv_indptr"],
                                          d["kv_indices"], d["last_page_len"], P, SCALE, causal=True)
    ctx_o, ctx_l = oracle.mla_attention(d["q_nope"], d["q_pe"], d["cache"], d["qo_indptr"], d["kv_indptr"],
                                        d["kv_indices"], d["last_page_len"], P, SCALE, causal=True,
                                        context_only=True)
    # own-token attention written out directly: query i sees own tokens 0..i
    qo = d["qo_indptr"]
    own_o = np.zeros_like(full_o)
    own_l = np.full(full_l.shape, -np.inf)
    for b in range(4):
        slots = _walk_slots(d["kv_indptr"], d["kv_indices"], d["last_page_len"], P, b)
        q_b = qo[b + 1] - qo[b]
        own = np.stack([d["cache"][pg, sl] for pg, sl in slots[len(slots) - q_b:]])  # [q_b, 576]
        for i in range(q_b):
            t = qo[b] + i
            q = np.concatenate([d["q_nope"][t], d["q_pe"][t]], axis=-1)
            s_ = (q @ own[: i + 1].T) * SCALE
            m = s_.max(axis=1, keepdims=True)
            e = np.exp(s_ - m)
            own_l[t] = (m + np.log(e.sum(axis=1, keepdims=True)))[:, 0]
            own_o[t] = (e / e.sum(axis=1, keepdims=True)) @ own[: i + 1, :D_C]
    mo, ml = oracle.merge_states(ctx_o, ctx_l, own_o, own_l)
    assert np.allclose(mo, full_o, rtol=0, atol=1e-12) and np.allclose(ml, full_l, rtol=0, atol=1e-12)
    # a row with no stored context attends nothing in context-only mode
    t = qo[2]
    assert np.all(ctx_o[t] == 0) and np.all(ctx_l[t] == -np.inf)
    with pytest.raises(ValueError):
        oracle.mla_attention(d["q_nope"][:3], d["q_pe"][:3], d["cache"], [0, 3], [0, 1], d["kv_indices"][:1],
                             [2], P, SCALE, context_only=True)


def check_kpe_zero_width(oracle):
    """Without a rope part (kpe width 0, flashinfer_mla_supports: kpe 0 or 64) the scores
    are q_nope . ckv alone: the same as the 576-wide form with q_pe = 0, whatever kpe
    holds; the output is still built from the 512 ckv columns."""
    d = _paged([3, 1, 5], [40, 70, 5], 2, 16, seed=31)
    z = np.zeros_like(d["q_pe"])
    o64, l64 = oracle.mla_attention(d["q_nope"], z, d["cache"], d["qo_indptr"], d["kv_indptr"], d["kv_indices"],
                                    d["last_page_len"], 16, SCALE)
    c512 = d["cache"][..., :D_C].copy()
    o0, l0 = oracle.mla_attention(d["q_nope"], d["q_pe"][..., :0], c512, d["qo_indptr"], d["kv_indptr"],
                                  d["kv_indices"], d["last_page_len"], 16, SCALE)
    assert np.allclose(o0, o64, rtol=0, atol=1e-13) and np.allclose(l0, l64, rtol=0, atol=1e-13)
    # and it differs from the rope form once q_pe is not zero
    o1, _ = oracle.mla_attention(d["q_nope"], d["q_pe"], d["cache"], d["qo_indptr"], d["kv_indptr"],
                                 d["kv_indices"], d["last_page_len"], 16, SCALE)
    assert not np.allclose(o1, o0, atol=1e-6)


ALL_CHECKS = [
    check_absorbed_equals_explicit,
    check_against_sdpa,
    check_golden_worked_example,
    check_closed_forms,
    check_single_visible_key,
    check_page_permutation,
    check_causal_noop_single_query,
    check_lse_merge,
    check_merge_closed_forms,
    check_empty_and_overhang,
    check_kv_lengths,
    check_append_slots,
    check_context_only_merge,
    check_kpe_zero_width,
]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(O)


# --------------------------------------------------------------------------- mutations
def _oracle_copy():
    spec = importlib.util.spec_from_file_location("mla_oracle_mut", O.__file__)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mut_start_aligned(mod):
    mod.visible_keys = lambda k, q, i, causal: (min(k, i + 1) if causal else k)


def _mut_drop_rope(mod):
    orig = mod.attend_one

    def f(q, keys, vis, sm_scale):
        q = q.copy()
        q[:, mod.KV_LORA_RANK:] = 0
        return orig(q, keys, vis, sm_scale)

    mod.attend_one = f


def _mut_wrong_scale(mod):
    orig = mod.attend_one
    mod.attend_one = lambda q, keys, vis, sm_scale: orig(q, keys, vis, 576 ** -0.5)


def _mut_log2_lse(mod):
    orig = mod.attend_one

    def f(q, keys, vis, sm_scale):
        o, l = orig(q, keys, vis, sm_scale)
        return o, l / math.log(2)

    mod.attend_one = f


def _mut_value_includes_rope(mod):
    # use the kpe tail in place of the first 64 ckv columns of the value
    orig = mod.attend_one

    def f(q, keys, vis, sm_scale):
        k2 = keys.copy()
        k2[:, :64] = keys[:, mod.KV_LORA_RANK:]
        o, l = orig(q, keys, vis, sm_scale)
        o2, _ = orig(q, k2, vis, sm_scale)
        return o2, l

    mod.attend_one = f


def _mut_kv_len_off_by_one(mod):
    orig = mod.kv_lengths

    def f(kv_indptr, last, page_size):
        n = np.asarray(kv_indptr)[1:] - np.asarray(kv_indptr)[:-1]
        return np.where(n > 0, n * page_size - np.asarray(last), 0)

    mod.kv_lengths = f


def _mut_slot_transposed(mod):
    def g(cache, kv_indptr, kv_indices, page_size, b, k_b):
        kv_indptr = np.asarray(kv_indptr)
        kv_indices = np.asarray(kv_indices)
        out = np.empty((k_b, np.asarray(cache).shape[-1]))
        for j in range(k_b):
            n = -(-k_b // page_size)
            # wrong: slot-major walk
            page = kv_indices[kv_indptr[b] + (j % n)]
            out[j] = np.asarray(cache)[page, (j // n) % page_size]
        return out

    mod.gather_row_keys = g


def _mut_merge_sign(mod):
    orig = mod.merge_states

    def f(oa, la, ob, lb):
        return orig(oa, -la, ob, -lb)

    mod.merge_states = f


def _mut_append_start_aligned(mod):
    # wrong: the step's tokens written at the start of the row instead of its end
    def f(cache, kv_new, qo_indptr, kv_indptr, kv_indices, last_page_len, page_size):
        out = mod._f64(cache).copy()
        new = mod._f64(kv_new)
        qo = mod._i64(qo_indptr)
        for b in range(len(qo) - 1):
            for i in range(int(qo[b + 1] - qo[b])):
                page, slot = mod.key_location(kv_indptr, kv_indices, page_size, b, i)
                out[page, slot] = new[qo[b] + i]
        return out

    mod.append_latent = f


def _mut_context_includes_own(mod):
    # wrong: a context-only query also sees the step's own tokens
    orig = mod.mla_attention

    def f(*a, context_only=False, **kw):
        return orig(*a, context_only=False, **{**kw, "causal": False}) if context_only else orig(*a, **kw)

    mod.mla_attention = f


MUTATIONS = [_mut_start_aligned, _mut_drop_rope, _mut_wrong_scale, _mut_log2_lse, _mut_value_includes_rope,
             _mut_kv_len_off_by_one, _mut_slot_transposed, _mut_merge_sign, _mut_append_start_aligned,
             _mut_context_includes_own]


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda m: m.__name__)
def test_pins_catch_planted_mistake(mutate):
    mod = _oracle_copy()
    mutate(mod)
    caught = []
    for check in ALL_CHECKS:
        try:
            check(mod)
        except Exception:
            caught.append(check.__name__)
    assert caught, f"no pin caught {mutate.__name__}"
