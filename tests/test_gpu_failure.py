"""Failure detection on the GPU without faulting anything.

Every wait inside the attention kernel is bounded.  A debug flag makes the kernel skip
its first key-tile load, so the wait for that tile never completes ("a flag that
nothing sets"): after the configured timeout the kernel records
MLA_ERR_DEVICE_TIMEOUT in the plan's status word (and its host-mapped copy), every
role unwinds, and mla_plan_check reports it.  The context stays usable: a normal run afterwards still
matches the oracle.
"""

import numpy as np
import pytest
import torch

import paged_head_latent_mla_b200 as M
from oracle import mla_oracle as O
from workloads import make_custom

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    from paged_head_latent_mla_b200 import _build

    _build.build()
    return M.load_library()


def _plan(d, **kw):
    return M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=d.num_heads,
                      page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, causal=d.causal, **kw)


def test_bounded_wait_reports_timeout_and_context_survives():
    dev = torch.device("cuda:0")
    d = make_custom([1, 3], [700, 300], 128, 64, seed=51)
    qn, qp, cache = d.q_nope.to(dev), d.q_pe.to(dev), d.cache.to(dev)
    plan = _plan(d, debug_flags=M.MLA_DEBUG_DROP_FIRST_KV_LOAD, wait_timeout_ns=50_000_000)
    M.mla_run(plan, qn, qp, cache, return_lse=True)
    assert M.mla_plan_check(plan) == M.MLA_ERR_DEVICE_TIMEOUT
    assert M.mla_plan_check(plan) == M.MLA_OK  # the status word was cleared
    # both copies of the word were cleared: the next failing run records and reports again
    M.mla_run(plan, qn, qp, cache)
    assert M.mla_plan_check(plan) == M.MLA_ERR_DEVICE_TIMEOUT
    assert M.mla_plan_check(plan) == M.MLA_OK
    plan.destroy()
    torch.cuda.synchronize(dev)  # no sticky CUDA error

    plan = _plan(d)
    out, lse = M.mla_run(plan, qn, qp, cache, return_lse=True)
    assert M.mla_plan_check(plan) == M.MLA_OK
    plan.destroy()
    ref_o, ref_l = O.mla_attention(d.q_nope, d.q_pe, d.cache, d.qo_indptr, d.kv_indptr, d.kv_indices,
                                   d.last_page_len, d.page_size, d.sm_scale, causal=d.causal)
    o = out.float().cpu().numpy()
    assert (np.abs(o - ref_o) <= 1e-2 + 1e-2 * np.abs(ref_o)).all()
    assert np.abs(lse.cpu().numpy() - ref_l).max() <= 1e-3


def test_launch_errors_are_status_codes_not_exceptions():
    dev = torch.device("cuda:0")
    d = make_custom([1], [100], 16, 16, seed=52)
    plan = _plan(d)
    lib = M.load_library()
    qn, qp, cache = d.q_nope.to(dev), d.q_pe.to(dev), d.cache.to(dev)
    out = torch.empty((1, 16, 512), dtype=torch.bfloat16, device=dev)
    # misaligned output pointer (TMA/vector stores need 16-byte alignment)
    st = lib.mla_run(plan.handle, qn.data_ptr(), qp.data_ptr(), cache.data_ptr(), out.data_ptr() + 2, None, None)
    assert st == M.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_run(plan.handle, None, qp.data_ptr(), cache.data_ptr(), out.data_ptr(), None, None) == \
        M.MLA_ERR_INVALID_ARGUMENT
    plan.destroy()


def test_status_slots_are_per_plan():
    """Each plan's host-mapped status copy is its own: with 150 plans alive (more than
    one 64-slot slab), a timeout in one is reported by that plan only, and every other
    plan reports OK; slots of destroyed plans are reused clean."""
    dev = torch.device("cuda:0")
    d = make_custom([1], [200], 16, 16, seed=53)
    qn, qp, cache = d.q_nope.to(dev), d.q_pe.to(dev), d.cache.to(dev)
    for _round in range(2):
        plans = [_plan(d) for _ in range(150)]
        bad = _plan(d, debug_flags=M.MLA_DEBUG_DROP_FIRST_KV_LOAD, wait_timeout_ns=50_000_000)
        plans.insert(75, bad)
        for p in plans:
            M.mla_run(p, qn, qp, cache)
        for p in plans:
            assert M.mla_plan_check(p) == (M.MLA_ERR_DEVICE_TIMEOUT if p is bad else M.MLA_OK)
        for p in plans:
            p.destroy()
    torch.cuda.synchronize(dev)
