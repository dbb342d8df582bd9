"""GPU test of mla_run_noalloc, the entry point for callers that may not allocate device
memory when they run attention (serving processes whose memory manager already owns
all of HBM, plug-in hosts without an allocator, loops where cudaMalloc would
synchronise the device).

It plans and runs a step with all of its device scratch in one fixed array inside the
library.  Each call is compared, through the C ABI, with the ordinary
mla_plan + mla_run path on the same inputs, within the parity tolerances used by the
other GPU tests, over several calls in a row (the array keeps the previous call's
contents, so stale state would show up here).  This file is named so that pytest
collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

import paged_head_latent_mla_b200 as M
from workloads import make_custom

pytestmark = pytest.mark.gpu

OUT_ATOL, OUT_RTOL, LSE_ATOL = 1e-2, 1e-2, 1e-3


@pytest.fixture(scope="module", autouse=True)
def lib():
    from paged_head_latent_mla_b200 import _build

    _build.build()
    return M.load_library()


def _case(kind):
    if kind == "long":  # long rows: split-KV partials in the fixed scratch, some unsplit
        return make_custom([1, 1, 1, 1, 2, 1], [20000, 18000, 21000, 900, 5000, 64], 128, 64, seed=41)
    if kind == "mixed":  # prefill tiles, ragged tails, an empty row, page size 16
        return make_custom([33, 1, 0, 5], [400, 1500, 10, 3], 16, 16, seed=42)
    raise KeyError(kind)


def _reference(d, dev):
    plan = M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=d.num_heads,
                      page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, causal=d.causal)
    out, lse = M.mla_run(plan, d.q_nope.to(dev), d.q_pe.to(dev), d.cache.to(dev), return_lse=True)
    assert M.mla_plan_check(plan) == M.MLA_OK
    plan.destroy()
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _noalloc(d, dev):
    qn, qp, cache = d.q_nope.to(dev), d.q_pe.to(dev), d.cache.to(dev)
    out = torch.full((d.total_tokens, d.num_heads, 512), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((d.total_tokens, d.num_heads), float("nan"), dtype=torch.float32, device=dev)
    M.mla_run_noalloc(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, qn, qp, cache, out, lse,
                      num_heads=d.num_heads, page_size=d.page_size, num_pages=d.num_pages,
                      sm_scale=d.sm_scale, causal=d.causal)
    torch.cuda.synchronize(dev)
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _assert_close(got, ref):
    (go, gl), (ro, rl) = got, ref
    err = np.abs(go - ro)
    assert (err <= OUT_ATOL + OUT_RTOL * np.abs(ro)).all(), f"out max err {err.max():.3e}"
    inf = np.isneginf(rl)
    assert np.array_equal(inf, np.isneginf(gl))
    if (~inf).any():
        assert np.abs(gl[~inf] - rl[~inf]).max() <= LSE_ATOL


def test_noalloc_matches_planned_path_over_consecutive_calls():
    dev = torch.device("cuda:0")
    cases = {k: _case(k) for k in ("long", "mixed")}
    refs = {k: _reference(d, dev) for k, d in cases.items()}
    # several calls in a row, alternating shapes, on the shared scratch array
    for k in ("long", "long", "mixed", "long"):
        _assert_close(_noalloc(cases[k], dev), refs[k])


def test_noalloc_rejects_steps_beyond_its_fixed_scratch():
    lib = M.load_library()
    n_ids = (1 << 19) + 1  # one page id more than the array has room for
    qo = np.array([0, 1], dtype=np.int32)
    kvp = np.array([0, n_ids], dtype=np.int32)
    kvi = np.zeros(n_ids, dtype=np.int32)
    last = np.array([64], dtype=np.int32)
    dims = M._Dims(128, 512, 64, 64, 1, 192 ** -0.5)
    p = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))  # noqa: E731
    st = lib.mla_run_noalloc(ctypes.byref(dims), 1, p(qo), p(kvp), p(kvi), p(last), 1, None, None, None, None,
                             None, None)
    assert st == M.MLA_ERR_INVALID_ARGUMENT
