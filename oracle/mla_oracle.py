"""Plain fp64 CPU oracle for batched paged latent attention (absorbed MLA).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product path (the CUDA library and its Python binding) never calls
it, and this module imports nothing from the product.

What it computes, and where the pages define it
-----------------------------------------------
Pages: "mstar.engine.resources.attn.flashinfer_mla" (module description;
``FlashInferMLAWrapper.run`` and ``.plan``; ``FlashInferMLAManager.run``),
"mstar.engine.resources.attn.ragged.wrappers" (``PrefixedPrefillWrapper``
class description), "mstar.engine.resources.attn.base"
(``AttentionManager.requires_kv_write``; ``captured_page_capacity``).

* The cache holds one latent row per token, ``[ckv | kpe]`` (512 + 64 wide), in
  fixed-size pages named by ``paged_kv_indptr`` / ``paged_kv_indices`` /
  ``paged_kv_last_page_len`` (flashinfer_mla page: module description and
  ``FlashInferMLAWrapper.plan``).
* The query arrives absorbed: ``q_nope`` is already multiplied by W_UK, so it is
  kv_lora_rank wide, and ``q_pe`` is used as given, with no rotation applied
  here (flashinfer_mla page: module description).
* Scores are ``(q_nope . ckv + q_pe . kpe) * sm_scale`` with the softmax scale of
  the original 192-wide head (flashinfer_mla page: ``FlashInferMLAWrapper``
  parameter ``sm_scale``).
* The output stays in latent space, ``[T, H, kv_lora_rank]``: the softmax
  weights applied to the ckv rows; W_UV is applied later by the layer
  (flashinfer_mla page: module description; ``FlashInferMLAWrapper.run``).
* With ``return_lse`` the call also returns the natural-log log-sum-exp of the
  (scaled) scores, ``[T, H]``, used to merge two key segments
  (flashinfer_mla page: ``FlashInferMLAManager.run``).
* Causal masking aligns each row's query block to the END of its keys
  (ragged.wrappers page: ``PrefixedPrefillWrapper``).  The step's own K/V is
  written to the cache before attention runs (base page:
  ``AttentionManager.requires_kv_write``), so the row's key count includes its
  own query tokens.

Readings where the pages are silent (each is listed in the design notes):
* kv length of a row with n pages: ``(n - 1) * page_size + last_page_len`` and 0
  for a row with no pages (the usual meaning of ``paged_kv_last_page_len``).
* A query that sees no key returns an all-zero output and lse = -inf (the
  identity of the LSE merge).
* Page ids may repeat within and across rows (shared prefixes; base page,
  ``captured_page_capacity``).

Everything here is the plain definition, in float64, summed in logical key
order.  No blocking, no online softmax, no reordering.
"""

from __future__ import annotations

import numpy as np

KV_LORA_RANK = 512
ROPE_DIM = 64
LATENT_DIM = KV_LORA_RANK + ROPE_DIM


def _f64(x) -> np.ndarray:
    """Exact conversion of any real array (including torch bf16 tensors) to float64."""
    try:
        import torch  # local import: torch is only needed to unwrap tensors

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _i64(x) -> np.ndarray:
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.int64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.int64)


def kv_lengths(kv_indptr, last_page_len, page_size: int) -> np.ndarray:
    """Keys held by each row: ``(n_b - 1) * page_size + last_page_len[b]``, or 0 when
    the row names no page (flashinfer_mla page, ``FlashInferMLAWrapper.plan`` inputs;
    ``FlashInferMLAManager.kv_len_buf``)."""
    kv_indptr = _i64(kv_indptr)
    last = _i64(last_page_len)
    n = kv_indptr[1:] - kv_indptr[:-1]
    return np.where(n > 0, (n - 1) * page_size + last, 0).astype(np.int64)


def key_location(kv_indptr, kv_indices, page_size: int, b: int, j: int) -> tuple[int, int]:
    """Physical (page id, slot) of logical key j of row b: the page is the
    ``j // page_size``-th entry of the row's page list, the slot ``j % page_size``."""
    kv_indptr = _i64(kv_indptr)
    kv_indices = _i64(kv_indices)
    return int(kv_indices[kv_indptr[b] + j // page_size]), int(j % page_size)


def gather_row_keys(cache, kv_indptr, kv_indices, page_size: int, b: int, k_b: int) -> np.ndarray:
    """The row's logical key sequence ``[k_b, 576]`` in float64, read page by page:
    logical key j is slot ``j % page_size`` of page ``kv_indices[kv_indptr[b] + j // page_size]``."""
    kv_indptr = _i64(kv_indptr)
    kv_indices = _i64(kv_indices)
    width = cache.shape[-1]
    if k_b == 0:
        return np.zeros((0, width))
    n_pages = -(-k_b // page_size)
    pages = kv_indices[kv_indptr[b] : kv_indptr[b] + n_pages]
    try:
        import torch

        if isinstance(cache, torch.Tensor):
            blk = cache[torch.from_numpy(pages)]
            return _f64(blk).reshape(n_pages * page_size, width)[:k_b]
    except ImportError:  # pragma: no cover
        pass
    blk = np.asarray(cache)[pages]
    return blk.astype(np.float64).reshape(n_pages * page_size, width)[:k_b]


def visible_keys(k_b: int, q_b: int, i: int, causal: bool) -> int:
    """Keys query i (0-based within its row) may attend.  Causal: end-aligned, so
    query i sees keys ``j <= k_b - q_b + i`` (ragged.wrappers page,
    ``PrefixedPrefillWrapper``), clamped to [0, k_b]."""
    if not causal:
        return int(k_b)
    return int(min(k_b, max(0, k_b - q_b + i + 1)))


def attend_one(q: np.ndarray, keys: np.ndarray, vis: int, sm_scale: float):
    """Attention of ``q [H, 576]`` over the first ``vis`` rows of ``keys [k, 576]``.

    Returns (out [H, 512], lse [H]) in float64: s_j = sm_scale * q . key_j,
    lse = log sum_j exp(s_j), out = sum_j exp(s_j - lse) * ckv_j.
    """
    H = q.shape[0]
    if vis == 0:
        return np.zeros((H, KV_LORA_RANK)), np.full(H, -np.inf)
    k = keys[:vis]
    s = (q @ k.T) * sm_scale  # [H, vis]
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    lse = (m + np.log(z))[:, 0]
    w = e / z
    out = w @ k[:, :KV_LORA_RANK]
    return out, lse


def mla_attention(
    q_nope,
    q_pe,
    cache,
    qo_indptr,
    kv_indptr,
    kv_indices,
    last_page_len,
    page_size: int,
    sm_scale: float,
    causal: bool = True,
    tokens=None,
    context_only: bool = False,
):
    """Paged absorbed-MLA attention, plain definition in float64.

    q_nope [T, H, 512], q_pe [T, H, 64], cache [num_pages, page_size, 576];
    returns out [T, H, 512] and lse [T, H] (natural log).  With ``tokens`` (an
    iterable of global token indices) only those tokens are computed; the other
    entries of the result are NaN.

    ``context_only``: every query of row b attends exactly the row's stored context,
    keys ``j < k_b - q_b`` (flashinfer_mla page, ``FlashInferMLAManager.kv_len_buf``:
    the planned length of a context-only row is its stored context, where its queries
    start); those keys precede every query, so no mask applies.  A row with
    ``q_b > k_b`` has no such context and is rejected.
    """
    qn = _f64(q_nope)
    qp = _f64(q_pe)
    qo_indptr = _i64(qo_indptr)
    kv_indptr = _i64(kv_indptr)
    kv_indices = _i64(kv_indices)
    T, H, _ = qn.shape
    B = len(qo_indptr) - 1
    k_all = kv_lengths(kv_indptr, last_page_len, page_size)
    q_full = np.concatenate([qn, qp], axis=-1)  # [T, H, 576]

    want = None if tokens is None else set(int(t) for t in tokens)
    out = np.full((T, H, KV_LORA_RANK), np.nan if want is not None else 0.0)
    lse = np.full((T, H), np.nan if want is not None else 0.0)
    for b in range(B):
        t0, t1 = int(qo_indptr[b]), int(qo_indptr[b + 1])
        if t1 == t0:
            continue
        if want is not None and not any(t in want for t in range(t0, t1)):
            continue
        k_b = int(k_all[b])
        q_b = t1 - t0
        if context_only:
            if k_b < q_b:
                raise ValueError(f"row {b}: {q_b} queries but only {k_b} keys (no stored context)")
            k_b -= q_b
        keys = gather_row_keys(cache, kv_indptr, kv_indices, page_size, b, k_b)
        for i in range(q_b):
            t = t0 + i
            if want is not None and t not in want:
                continue
            vis = k_b if context_only else visible_keys(k_b, q_b, i, causal)
            out[t], lse[t] = attend_one(q_full[t], keys, vis, sm_scale)
    return out, lse


def merge_states(out_a, lse_a, out_b, lse_b):
    """Combine attention over two disjoint key sets from their outputs and natural
    log-sum-exps (flashinfer_mla page, ``FlashInferMLAManager.run``: the lse is
    returned for merging with another key segment).

    out = (e^{lse_a} out_a + e^{lse_b} out_b) / (e^{lse_a} + e^{lse_b}),
    lse = log(e^{lse_a} + e^{lse_b}); an empty segment (lse = -inf) contributes nothing.
    """
    out_a, lse_a, out_b, lse_b = map(_f64, (out_a, lse_a, out_b, lse_b))
    m = np.maximum(lse_a, lse_b)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    wa = np.exp(lse_a - m_safe)
    wb = np.exp(lse_b - m_safe)
    z = wa + wb
    with np.errstate(invalid="ignore", divide="ignore"):
        out = (wa[..., None] * out_a + wb[..., None] * out_b) / z[..., None]
        lse = m_safe + np.log(z)
    empty = z == 0
    out = np.where(empty[..., None], 0.0, out)
    lse = np.where(empty, -np.inf, lse)
    return out, lse


def merge_many(outs, lses):
    """Merge any number of key segments by LSE: M = max lse_i,
    out = sum_i e^{lse_i - M} out_i / sum_i e^{lse_i - M}, lse = M + log sum_i e^{lse_i - M}."""
    outs = np.stack([_f64(o) for o in outs])
    lses = np.stack([_f64(l) for l in lses])
    m = lses.max(axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lses - m_safe)
    z = w.sum(axis=0)
    with np.errstate(invalid="ignore", divide="ignore"):
        out = (w[..., None] * outs).sum(axis=0) / z[..., None]
        lse = m_safe + np.log(z)
    empty = z == 0
    return np.where(empty[..., None], 0.0, out), np.where(empty, -np.inf, lse)


def append_latent(cache, kv_new, qo_indptr, kv_indptr, kv_indices, last_page_len, page_size: int):
    """The step's latent rows written into their cache slots (base page,
    ``AttentionManager.requires_kv_write``: the layer writes the step's K/V before the
    attention runs, so the row's keys end with its own tokens).

    Token i of row b (global token ``qo_indptr[b] + i``) is logical key
    ``k_b - q_b + i`` of its row; ``kv_new [T, 576]`` row t is stored at that key's
    (page, slot).  Returns a float64 copy of ``cache`` with those rows replaced.

    Page ids may repeat (reading of ``captured_page_capacity`` on the base page), so
    two tokens can name one slot; the write then leaves one of their rows there, and
    which one is not fixed by the method.  This copy writes in token order, so it
    holds the later token's row: one valid result among several, and a check against
    it must accept any of the rows that name the slot.  A row with ``q_b > k_b`` has
    no slot for its first tokens and is rejected.
    """
    out = _f64(cache).copy()
    new = _f64(kv_new)
    qo_indptr = _i64(qo_indptr)
    k_all = kv_lengths(kv_indptr, last_page_len, page_size)
    for b in range(len(qo_indptr) - 1):
        t0, t1 = int(qo_indptr[b]), int(qo_indptr[b + 1])
        q_b, k_b = t1 - t0, int(k_all[b])
        if q_b > k_b:
            raise ValueError(f"row {b}: {q_b} new tokens but only {k_b} keys in its pages")
        for i in range(q_b):
            page, slot = key_location(kv_indptr, kv_indices, page_size, b, k_b - q_b + i)
            out[page, slot] = new[t0 + i]
    return out
