"""GPU tests of mla_run_noalloc, the entry point for callers that may not allocate device
memory when they run attention: serving processes whose memory manager already owns
all of HBM, plug-in hosts that give the library no allocator, and loops where a
cudaMalloc or cudaFree could synchronise the device.

The call plans and runs a step with all of its device scratch in one fixed array inside
the library.  Each call's output is compared, through the C ABI, with the fp64 oracle
on the same seeded inputs, at the parity tolerances of the other GPU tests, over several
calls in a row (the array keeps the previous call's contents, so stale state would show
up here), with and without a rope part.  The tests also check that the calls leave the
device's memory use unchanged, that a capturing stream is refused, and that the status
word the call hands back reads 0.  This file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

import paged_head_latent_mla_b200 as M
from oracle import mla_oracle as O
from workloads import make_custom

pytestmark = pytest.mark.gpu

OUT_ATOL, OUT_RTOL, LSE_ATOL = 1e-2, 1e-2, 1e-3
DEV = torch.device("cuda:0")


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
    if kind == "kpe0":  # no rope part: 512-wide cache rows, no q_pe
        return make_custom([1, 4, 1], [9000, 300, 2600], 64, 32, seed=43)
    raise KeyError(kind)


def _inputs(kind, d):
    """Device inputs of a case (the kpe-0 case drops the rope columns)."""
    if kind == "kpe0":
        return d.q_nope.to(DEV), None, d.cache[..., :512].contiguous().to(DEV), 0
    return d.q_nope.to(DEV), d.q_pe.to(DEV), d.cache.to(DEV), 64


def _oracle(kind, d):
    if kind == "kpe0":
        return O.mla_attention(d.q_nope, d.q_pe[..., :0], d.cache[..., :512], d.qo_indptr, d.kv_indptr,
                               d.kv_indices, d.last_page_len, d.page_size, d.sm_scale, causal=d.causal)
    return O.mla_attention(d.q_nope, d.q_pe, d.cache, d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len,
                           d.page_size, d.sm_scale, causal=d.causal)


def _noalloc(d, inputs, out, lse, status):
    qn, qp, cache, rope = inputs
    out.fill_(float("nan"))
    lse.fill_(float("nan"))
    status.fill_(-1)
    M.mla_run_noalloc(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, qn, qp, cache, out, lse,
                      num_heads=d.num_heads, page_size=d.page_size, num_pages=d.num_pages,
                      sm_scale=d.sm_scale, causal=d.causal, rope_dim=rope, status=status)
    torch.cuda.synchronize(DEV)
    # copied to the host before any conversion, so reading the results allocates no
    # device memory either
    return out.cpu().float().numpy(), lse.cpu().numpy(), int(status.cpu().item())


def _assert_close(go, gl, ref):
    ro, rl = ref
    err = np.abs(go - ro)
    assert (err <= OUT_ATOL + OUT_RTOL * np.abs(ro)).all(), f"out max err {err.max():.3e}"
    inf = np.isneginf(rl)
    assert np.array_equal(inf, np.isneginf(gl))
    if (~inf).any():
        assert np.abs(gl[~inf] - rl[~inf]).max() <= LSE_ATOL


def test_noalloc_matches_oracle_over_consecutive_calls():
    kinds = ("long", "mixed", "kpe0")
    cases = {k: _case(k) for k in kinds}
    refs = {k: _oracle(k, d) for k, d in cases.items()}
    inputs = {k: _inputs(k, d) for k, d in cases.items()}
    bufs = {k: (torch.empty((d.total_tokens, d.num_heads, 512), dtype=torch.bfloat16, device=DEV),
                torch.empty((d.total_tokens, d.num_heads), dtype=torch.float32, device=DEV))
            for k, d in cases.items()}
    status = torch.empty(1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize(DEV)
    order = ("long", "long", "mixed", "kpe0", "long", "kpe0", "mixed")
    # one unchecked pass first: the first call's one-time set-up, and the first use of
    # every kernel involved (lazily loaded code takes device memory once)
    for k in kinds:
        _noalloc(cases[k], inputs[k], *bufs[k], status)
    torch.cuda.synchronize(DEV)
    free0, _ = torch.cuda.mem_get_info(DEV)
    alloc0 = torch.cuda.memory_allocated(DEV)
    # several calls in a row, alternating shapes, on the shared scratch array
    for k in order:
        go, gl, st = _noalloc(cases[k], inputs[k], *bufs[k], status)
        assert st == M.MLA_OK, f"{k}: device status {st:#x}"
        _assert_close(go, gl, refs[k])
    free1, _ = torch.cuda.mem_get_info(DEV)
    assert torch.cuda.memory_allocated(DEV) == alloc0
    assert free1 == free0, f"device free memory moved by {free0 - free1} bytes"


def test_noalloc_refuses_a_capturing_stream():
    d = _case("mixed")
    qn, qp, cache, rope = _inputs("mixed", d)
    out = torch.empty((d.total_tokens, d.num_heads, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((d.total_tokens, d.num_heads), dtype=torch.float32, device=DEV)
    s = torch.cuda.Stream(DEV)
    g = torch.cuda.CUDAGraph()
    err = None
    with torch.cuda.graph(g, stream=s):
        out.zero_()  # the captured graph is not empty
        try:
            M.mla_run_noalloc(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, qn, qp, cache, out, lse,
                              num_heads=d.num_heads, page_size=d.page_size, num_pages=d.num_pages,
                              sm_scale=d.sm_scale, causal=d.causal, stream=s.cuda_stream)
        except M.MlaError as e:
            err = e
    assert err is not None and err.status == M.MLA_ERR_UNSUPPORTED
    del g
    torch.cuda.synchronize(DEV)


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
                             None, None, None)
    assert st == M.MLA_ERR_INVALID_ARGUMENT
