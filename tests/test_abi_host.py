"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports every
function include/mla.h declares, validates inputs with the documented status codes,
and plans on the host."""

import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

import paged_head_latent_mla_b200 as M  # noqa: E402
from workloads import make_config  # noqa: E402

SCALE = 192 ** -0.5


@pytest.fixture(scope="module", autouse=True)
def built_library():
    from paged_head_latent_mla_b200 import _build

    _build.build()
    return M.load_library()


def declared_functions():
    with open(os.path.join(ROOT, "include", "mla.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(mla_[a-z_]+)\s*\(", text)
    return sorted(set(names))


def test_exports_every_declared_function():
    lib = M.load_library()
    names = declared_functions()
    assert set(names) == set(M.EXPORTED), names
    for n in names:
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_supports_matrix():
    assert M.mla_supports(512, 64, 128, 64)
    for H in (16, 32, 64, 128):
        for P in (16, 32, 64, 128):
            assert M.mla_supports(512, 64, H, P)
    assert M.mla_supports(512, 0, 128, 64)  # kpe 0 or 64 (flashinfer_mla_supports)
    assert not M.mla_supports(512, 32, 128, 64)
    assert not M.mla_supports(256, 64, 128, 64)
    assert not M.mla_supports(512, 64, 8, 64)
    assert not M.mla_supports(512, 64, 128, 1)
    assert not M.mla_supports(512, 64, 128, 48)


def test_status_strings():
    for code in range(6):
        assert M.status_string(code)
    assert M.status_string(99) == "unknown status"


def _plan(**kw):
    args = dict(qo_indptr=[0, 1, 3], kv_indptr=[0, 2, 5], kv_indices=[0, 1, 2, 3, 4], last_page_len=[5, 16],
                num_heads=16, page_size=16, num_pages=8, sm_scale=SCALE, host_only=True)
    args.update(kw)
    return M.mla_plan(**args)


def test_host_plan_basic():
    p = _plan()
    d = M.mla_plan_describe(p)
    assert list(d["kv_len"]) == [21, 48]
    assert d["info"]["total_tokens"] == 3
    assert d["info"]["num_sms"] == 148
    p.destroy()


@pytest.mark.parametrize(
    "bad",
    [
        dict(qo_indptr=[1, 1, 3]),  # [0] != 0
        dict(qo_indptr=[0, 2, 1]),  # decreasing
        dict(kv_indptr=[0, 3, 2]),
        dict(kv_indices=[0, 1, 2, 3, 8]),  # page id out of range
        dict(kv_indices=[0, 1, 2, 3, -1]),
        dict(last_page_len=[0, 16]),  # row with pages needs >= 1
        dict(last_page_len=[5, 17]),
        dict(num_pages=0),
        dict(split_keys=100),  # not a multiple of the key tile
        dict(sm_scale=float("nan")),
    ],
)
def test_invalid_arguments(bad):
    with pytest.raises(M.MlaError) as e:
        _plan(**bad)
    assert e.value.status == M.MLA_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("bad", [dict(num_heads=8), dict(page_size=8), dict(kv_lora_rank=256),
                                 dict(rope_dim=32), dict(num_heads=96)])
def test_unsupported_shapes(bad):
    with pytest.raises(M.MlaError) as e:
        _plan(**bad)
    assert e.value.status == M.MLA_ERR_UNSUPPORTED


def test_empty_row_may_have_zero_last_page_len():
    p = _plan(kv_indptr=[0, 0, 3], kv_indices=[0, 1, 2], last_page_len=[0, 4])
    assert list(M.mla_plan_describe(p)["kv_len"]) == [0, 36]


def test_null_pointers_rejected_by_c_abi():
    lib = M.load_library()
    out = ctypes.c_void_p()
    st = lib.mla_plan(None, 0, None, None, None, None, 1, None, None, ctypes.byref(out))
    assert st == M.MLA_ERR_INVALID_ARGUMENT and not out.value
    st = lib.mla_plan(ctypes.byref(M._Dims(16, 512, 64, 16, 4, SCALE)), 1, None, None, None, None, 1, None,
                      ctypes.byref(M._Options(0, 0, 0, 0, 1)), ctypes.byref(out))
    assert st == M.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_plan_check(None) == M.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_run(None, None, None, None, None, None, None) == M.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_plan_update(None, 0, None, None, None, None, None, None) == M.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_append_kv(None, None, None, None) == M.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_run_append(None, None, None, None, None, None, None, None) == M.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_merge_state(None, None, None, None, None, None, 4, None) == M.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_merge_state(None, None, None, None, None, None, -1, None) == M.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_merge_state(None, None, None, None, None, None, 0, None) == M.MLA_OK  # nothing to do
    lib.mla_plan_destroy(None)  # no-op


def test_host_only_plan_cannot_run():
    p = _plan()
    lib = M.load_library()
    assert lib.mla_run(p.handle, None, None, None, None, None, None) == M.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_plan_check(p.handle) == M.MLA_OK


def test_plain_c_client(tmp_path):
    """include/mla.h is a C header: a C99 program compiles against it with warnings as
    errors, links the library, and drives a host-only plan through the ABI."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(M.LIB_PATH)
    exe = str(tmp_path / "abi_client")
    cmd = [cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_client.c"), "-L", lib_dir, "-l:libmla_b200.so",
           "-Wl,-rpath," + lib_dir, "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    got = dict((line.split(" ", 1) + [""])[:2] for line in r.stdout.strip().splitlines())
    assert got["supports"] == "1 1 0"
    assert got["plan"] == "0 ok"
    assert got["info"] == "0 batch 2 tokens 4 work 4 merge 1"  # the 3-tile row split for latency
    assert got["kv_len"] == "0 37 150"
    assert got["update_same"] == "0 1"
    assert got["update_changed"] == "0 0"
    assert got["update_bad"] == str(M.MLA_ERR_INVALID_ARGUMENT)
    assert got["run_host_only"] == str(M.MLA_ERR_INVALID_ARGUMENT)
    assert got["merge_state_bad"] == str(M.MLA_ERR_INVALID_ARGUMENT)
    assert "done" in got


def test_cache_shape_checked_before_any_launch():
    """The binding refuses a cache tensor with fewer pages than the plan declares, another
    page size or another row width before it reaches the library (the kernels' tensor
    maps span num_pages * page_size rows, so a smaller tensor would be read past its
    end).  Checked with CPU tensors: the shape check comes before the device checks."""
    import torch

    d = make_config("tiny_decode", tables_only=True)
    p = M.mla_plan(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, num_heads=d.num_heads,
                   page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale, host_only=True)
    T, H = int(d.qo_indptr[-1]), d.num_heads
    qn = torch.zeros((T, H, 512), dtype=torch.bfloat16)
    qp = torch.zeros((T, H, 64), dtype=torch.bfloat16)
    for shape in [(d.num_pages - 1, d.page_size, 576), (d.num_pages, d.page_size * 2, 576),
                  (d.num_pages, d.page_size, 512), (d.num_pages * d.page_size, 576)]:
        cache = torch.zeros(shape, dtype=torch.bfloat16)
        with pytest.raises(ValueError, match="cache must have shape"):
            M.mla_run(p, qn, qp, cache)
        with pytest.raises(ValueError, match="cache must have shape"):
            M.mla_append_kv(p, torch.zeros((T, 576), dtype=torch.bfloat16), cache)
        with pytest.raises(ValueError, match="cache must have shape"):
            M.mla_run_noalloc(d.qo_indptr, d.kv_indptr, d.kv_indices, d.last_page_len, qn, qp, cache,
                              torch.zeros((T, H, 512), dtype=torch.bfloat16), num_heads=H,
                              page_size=d.page_size, num_pages=d.num_pages, sm_scale=d.sm_scale)
    p.destroy()


def _write_tables(path, steps):
    """One or two steps' tables in the int32 layout tests/c/plan_timer.cpp reads."""
    with open(path, "wb") as f:
        for d in steps:
            hdr = np.array([d.num_heads, d.page_size, d.num_pages, d.batch, 1 if d.causal else 0], np.int32)
            for a in (hdr, d.qo_indptr.numpy(), d.kv_indptr.numpy(), d.kv_indices.numpy(), d.last_page_len.numpy()):
                f.write(np.ascontiguousarray(a, dtype=np.int32).tobytes())


def test_plan_timer_cpp_client(tmp_path):
    """The C++ planning timer (the same client the benchmark runs on the GPU machine) builds
    against include/mla.h, links the library and times host-only plans of the batch-64
    decode step: fresh plans, unchanged updates (recognised, nothing re-planned) and
    changed updates.  The numbers are reported, not asserted: this host is not the
    benchmark's."""
    import shutil
    import subprocess

    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    lib_dir = os.path.dirname(M.LIB_PATH)
    exe = str(tmp_path / "plan_timer")
    r = subprocess.run([cxx, "-O2", "-std=c++17", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c", "plan_timer.cpp"), "-L", lib_dir, "-l:libmla_b200.so",
                        "-Wl,-rpath," + lib_dir, "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    tables = str(tmp_path / "decode_b64.tables")
    _write_tables(tables, [make_config("decode_b64", tables_only=True),
                           make_config("decode_b64", seed=1, tables_only=True)])
    r = subprocess.run([exe, tables, "50", "1"], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    got = {k: float(v) for k, v in (line.split() for line in r.stdout.strip().splitlines())}
    assert set(got) == {"fresh", "update_same", "update_changed"}
    assert all(v > 0 for v in got.values())
    assert got["update_same"] < got["update_changed"]  # an unchanged step is only compared
    print("host-only planning, decode_b64 (us):", got)


def test_e2e_cpp_client_builds(tmp_path):
    """The C++ end-to-end client that the benchmark times on the GPU (plan, upload, run,
    download, pipelined two deep through the C ABI) compiles warning-free against
    include/mla.h and the CUDA runtime and links the library; without a GPU it is only
    built, and it refuses a missing argument list."""
    import shutil
    import subprocess

    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    if not os.path.exists(os.path.join(cuda, "include", "cuda_runtime.h")):
        pytest.skip("no CUDA runtime headers")
    lib_dir = os.path.dirname(M.LIB_PATH)
    exe = str(tmp_path / "e2e_driver")
    r = subprocess.run([cxx, "-O2", "-std=c++17", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I",
                        os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c", "e2e_driver.cpp"), "-L",
                        lib_dir, "-l:libmla_b200.so", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                        "-Wl,-rpath," + lib_dir + ":" + os.path.join(cuda, "lib64"), "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 2 and "usage" in r.stderr
