"""Python binding of the sm_100a paged latent-attention library (``libmla_b200.so``).

Argument marshalling only: torch tensors give device pointers and the current CUDA
stream; host index tables are copied into int32 arrays.  Every step of the attention
runs in the library's CUDA kernels.  If the library is missing the calls raise; there
is no other implementation to fall back to.

Names follow the C ABI in ``include/mla.h``: ``mla_supports``, ``mla_plan``,
``mla_plan_update``, ``mla_run``, ``mla_append_kv``, ``mla_run_append``,
``mla_merge_state``, ``mla_plan_check``, ``mla_plan_get_info``, ``mla_plan_describe``,
``mla_plan_kernel_times``, ``mla_run_noalloc``, ``mla_plan_destroy``,
``mla_status_string``.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla_b200.so")

MLA_OK = 0
MLA_ERR_INVALID_ARGUMENT = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_CUDA = 3
MLA_ERR_OUT_OF_MEMORY = 4
MLA_ERR_DEVICE_TIMEOUT = 5
MLA_KEY_TILE = 64  # keys per kernel tile; split sizes are multiples of it
MLA_DEBUG_DROP_FIRST_KV_LOAD = 1
MLA_DEBUG_KERNEL_TIMING = 2
WORK_FIELDS = 8
MERGE_FIELDS = 4
KV_LORA_RANK = 512
ROPE_DIM = 64

EXPORTED = (
    "mla_supports",
    "mla_plan",
    "mla_plan_update",
    "mla_run",
    "mla_append_kv",
    "mla_run_append",
    "mla_merge_state",
    "mla_plan_check",
    "mla_plan_get_info",
    "mla_plan_describe",
    "mla_plan_kernel_times",
    "mla_run_noalloc",
    "mla_plan_destroy",
    "mla_status_string",
)


class MlaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class _Dims(ctypes.Structure):
    _fields_ = [
        ("num_heads", ctypes.c_int32),
        ("kv_lora_rank", ctypes.c_int32),
        ("rope_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("sm_scale", ctypes.c_float),
    ]


class _Options(ctypes.Structure):
    _fields_ = [
        ("split_keys", ctypes.c_int32),
        ("num_sms", ctypes.c_int32),
        ("wait_timeout_ns", ctypes.c_uint64),
        ("debug_flags", ctypes.c_int32),
        ("host_only", ctypes.c_int32),
        ("graph_max_batch", ctypes.c_int32),
        ("graph_max_tokens", ctypes.c_int32),
        ("graph_max_page_ids", ctypes.c_int32),
        ("context_only", ctypes.c_int32),
        ("cascade", ctypes.c_int32),
    ]


class _Info(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("total_tokens", ctypes.c_int32),
        ("num_work", ctypes.c_int32),
        ("num_merge", ctypes.c_int32),
        ("num_partials", ctypes.c_int32),
        ("num_sms", ctypes.c_int32),
        ("workspace_bytes", ctypes.c_int64),
        ("num_merge_refs", ctypes.c_int32),
        ("num_cascade", ctypes.c_int32),
        ("graph", ctypes.c_int32),
        ("work_capacity", ctypes.c_int32),
    ]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load (once) and return the library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"CUDA library {path} is missing: build it with "
            "`python -m paged_head_latent_mla_b200._build` (there is no fallback)")
    lib = ctypes.CDLL(path)
    vp = ctypes.c_void_p
    i32p = vp  # host int32 tables and out-arrays travel as addresses (see _ptr)
    lib.mla_supports.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.mla_supports.restype = ctypes.c_int
    lib.mla_plan.argtypes = [ctypes.POINTER(_Dims), ctypes.c_int32, i32p, i32p, i32p, i32p, ctypes.c_int32, vp,
                             ctypes.POINTER(_Options), ctypes.POINTER(vp)]
    lib.mla_plan.restype = ctypes.c_int
    lib.mla_run.argtypes = [vp, vp, vp, vp, vp, vp, vp]
    lib.mla_run.restype = ctypes.c_int
    lib.mla_plan_update.argtypes = [vp, ctypes.c_int32, i32p, i32p, i32p, i32p, vp, i32p]
    lib.mla_plan_update.restype = ctypes.c_int
    lib.mla_append_kv.argtypes = [vp, vp, vp, vp]
    lib.mla_append_kv.restype = ctypes.c_int
    lib.mla_run_append.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp]
    lib.mla_run_append.restype = ctypes.c_int
    lib.mla_merge_state.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_int64, vp]
    lib.mla_merge_state.restype = ctypes.c_int
    lib.mla_plan_check.argtypes = [vp]
    lib.mla_plan_check.restype = ctypes.c_int
    lib.mla_plan_get_info.argtypes = [vp, ctypes.POINTER(_Info)]
    lib.mla_plan_get_info.restype = ctypes.c_int
    lib.mla_plan_describe.argtypes = [vp, i32p, i32p, i32p, i32p]
    lib.mla_plan_describe.restype = ctypes.c_int
    fp = ctypes.POINTER(ctypes.c_float)
    lib.mla_plan_kernel_times.argtypes = [vp, ctypes.c_int32, fp, fp, i32p]
    lib.mla_plan_kernel_times.restype = ctypes.c_int
    lib.mla_run_noalloc.argtypes = [ctypes.POINTER(_Dims), ctypes.c_int32, i32p, i32p, i32p, i32p, ctypes.c_int32,
                                    vp, vp, vp, vp, vp, vp, vp]
    lib.mla_run_noalloc.restype = ctypes.c_int
    lib.mla_plan_destroy.argtypes = [vp]
    lib.mla_plan_destroy.restype = None
    lib.mla_status_string.argtypes = [ctypes.c_int]
    lib.mla_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().mla_status_string(int(status)).decode()


mla_status_string = status_string


def _i32(x) -> np.ndarray:
    if type(x) is np.ndarray and x.dtype == np.int32 and x.flags.c_contiguous:
        return x  # already what the library reads
    try:
        import torch

        if isinstance(x, torch.Tensor):
            if x.is_cuda:
                raise ValueError("page tables are host arrays (CPU tensors, numpy arrays or lists)")
            x = x.numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a: np.ndarray) -> int:
    """Address of a host int32 array's data, for the table arguments (declared void*)."""
    return a.ctypes.data


def mla_supports(kv_lora_rank: int, rope_dim: int, num_heads: int, page_size: int) -> bool:
    return bool(load_library().mla_supports(kv_lora_rank, rope_dim, num_heads, page_size))


class MlaPlan:
    """Owns one C plan handle (``mla_plan_t``); destroyed with the object."""

    def __init__(self, handle: int, batch: int, num_heads: int, total_tokens: int, graph_max_tokens: int = 0,
                 rope_dim: int = ROPE_DIM, num_pages: int = 0, page_size: int = 0):
        self._h = ctypes.c_void_p(handle)
        self.batch = batch
        self.num_heads = num_heads
        self.total_tokens = total_tokens
        self.rope_dim = rope_dim
        # the cache every run of this plan reads is [num_pages, page_size, 512 + rope_dim]
        self.num_pages = num_pages
        self.page_size = page_size
        # a graph plan's per-token buffers hold graph_max_tokens tokens
        self.graph_max_tokens = graph_max_tokens

    @property
    def token_capacity(self) -> int:
        """Tokens every per-token buffer passed with this plan must hold."""
        return self.graph_max_tokens if self.graph_max_tokens > 0 else self.total_tokens

    @property
    def handle(self) -> ctypes.c_void_p:
        if not self._h:
            raise RuntimeError("plan was destroyed")
        return self._h

    def destroy(self) -> None:
        if self._h:
            load_library().mla_plan_destroy(self._h)
            self._h = ctypes.c_void_p(None)

    def __del__(self):  # pragma: no cover - interpreter shutdown order
        try:
            self.destroy()
        except Exception:
            pass


def mla_plan(qo_indptr, kv_indptr, kv_indices, last_page_len, *, num_heads: int, page_size: int, num_pages: int,
             sm_scale: float, causal: bool = True, kv_lora_rank: int = KV_LORA_RANK, rope_dim: int = ROPE_DIM,
             split_keys: int = 0, num_sms: int = 0, wait_timeout_ns: int = 0, debug_flags: int = 0,
             host_only: bool = False, graph_max_batch: int = 0, graph_max_tokens: int = 0,
             graph_max_page_ids: int = 0, context_only: bool = False, cascade: bool = False,
             stream=None) -> MlaPlan:
    """Plan one step from host page tables (``mla_plan``).  ``graph_max_*`` make a graph
    plan for a bucket (fixed device buffers and launch shapes, re-planned in place by
    ``mla_plan_update``); ``context_only`` attends only each row's stored context;
    ``cascade`` attends prefixes shared by consecutive rows once per group."""
    lib = load_library()
    qo = _i32(qo_indptr)
    kvp = _i32(kv_indptr)
    kvi = _i32(kv_indices)
    last = _i32(last_page_len)
    batch = len(qo) - 1
    if batch < 0 or len(kvp) != batch + 1 or len(last) != batch:
        raise MlaError(MLA_ERR_INVALID_ARGUMENT, "mla_plan: table lengths")
    if len(kvi) < int(kvp[-1]):
        raise MlaError(MLA_ERR_INVALID_ARGUMENT, "mla_plan: kv_indices shorter than kv_indptr[-1]")
    dims = _Dims(num_heads, kv_lora_rank, rope_dim, page_size, num_pages, sm_scale)
    opts = _Options(split_keys, num_sms, wait_timeout_ns, debug_flags, 1 if host_only else 0, graph_max_batch,
                    graph_max_tokens, graph_max_page_ids, 1 if context_only else 0, 1 if cascade else 0)
    if stream is None and not host_only:
        import torch

        stream = torch.cuda.current_stream().cuda_stream
    out = ctypes.c_void_p()
    kvi_arr = kvi if len(kvi) else np.zeros(1, dtype=np.int32)
    st = lib.mla_plan(ctypes.byref(dims), batch, _ptr(qo), _ptr(kvp), _ptr(kvi_arr), _ptr(last),
                      1 if causal else 0, ctypes.c_void_p(stream or 0), ctypes.byref(opts), ctypes.byref(out))
    if st != MLA_OK:
        raise MlaError(st, "mla_plan")
    return MlaPlan(out.value, batch, num_heads, int(qo[-1]), graph_max_tokens if graph_max_tokens > 0 else 0,
                   rope_dim, num_pages, page_size)


def mla_plan_update(plan: MlaPlan, qo_indptr, kv_indptr, kv_indices, last_page_len, stream=None) -> bool:
    """Re-plan ``plan`` in place for another step (``mla_plan_update``).  Returns True
    when the tables equal the plan's current step and nothing was done."""
    lib = load_library()
    qo = _i32(qo_indptr)
    kvp = _i32(kv_indptr)
    kvi = _i32(kv_indices)
    last = _i32(last_page_len)
    batch = len(qo) - 1
    if batch < 0 or len(kvp) != batch + 1 or len(last) != batch or len(kvi) < int(kvp[-1]):
        raise MlaError(MLA_ERR_INVALID_ARGUMENT, "mla_plan_update: table lengths")
    if stream is None:
        import torch

        stream = torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else 0
    kvi_arr = kvi if len(kvi) else np.zeros(1, dtype=np.int32)
    last_arr = last if len(last) else np.zeros(1, dtype=np.int32)
    reused = ctypes.c_int32(0)
    st = lib.mla_plan_update(plan.handle, batch, _ptr(qo), _ptr(kvp), _ptr(kvi_arr), _ptr(last_arr),
                             ctypes.c_void_p(stream or 0), ctypes.byref(reused))
    if st != MLA_OK:
        raise MlaError(st, "mla_plan_update")
    plan.batch = batch
    plan.total_tokens = int(qo[-1])
    return bool(reused.value)


def mla_plan_get_info(plan: MlaPlan) -> dict:
    info = _Info()
    st = load_library().mla_plan_get_info(plan.handle, ctypes.byref(info))
    if st != MLA_OK:
        raise MlaError(st, "mla_plan_get_info")
    return {f: getattr(info, f) for f, _ in _Info._fields_}


def mla_plan_describe(plan: MlaPlan) -> dict:
    """kv_len [B], work [num_work, 8], merge [num_merge, 4] and the merge reference list
    refs [num_merge_refs] as int32 arrays."""
    info = mla_plan_get_info(plan)
    kv_len = np.zeros(max(1, info["batch"]), dtype=np.int32)
    work = np.zeros((max(1, info["num_work"]), WORK_FIELDS), dtype=np.int32)
    merge = np.zeros((max(1, info["num_merge"]), MERGE_FIELDS), dtype=np.int32)
    refs = np.zeros(max(1, info["num_merge_refs"]), dtype=np.int32)
    st = load_library().mla_plan_describe(plan.handle, _ptr(kv_len), _ptr(work), _ptr(merge), _ptr(refs))
    if st != MLA_OK:
        raise MlaError(st, "mla_plan_describe")
    return {
        "kv_len": kv_len[: info["batch"]],
        "work": work[: info["num_work"]],
        "merge": merge[: info["num_merge"]],
        "refs": refs[: info["num_merge_refs"]],
        "info": info,
    }


def _check_cache_shape(cache, num_pages: int, page_size: int, rope_dim: int) -> None:
    """The cache must be [>= num_pages, page_size, 512 + rope_dim]: the kernels' tensor
    maps span num_pages * page_size rows of 512 + rope_dim columns, so a tensor with
    fewer pages would be read past its end (a larger pool is fine)."""
    width = KV_LORA_RANK + rope_dim
    shape = tuple(getattr(cache, "shape", ()))
    if len(shape) != 3 or shape[1] != page_size or shape[2] != width or shape[0] < num_pages:
        raise ValueError(f"cache must have shape (>= {num_pages}, {page_size}, {width}) "
                         f"(num_pages, page_size, 512 + rope_dim), got {shape}")


def _check_dev_tensor(t, name, dtype, shape):
    import torch

    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def mla_run(plan: MlaPlan, q_nope, q_pe, cache, out=None, lse=None, return_lse: bool = False, stream=None,
            kv_new=None):
    """Run the planned attention (``mla_run``).  Returns ``out`` or ``(out, lse)``.
    With ``kv_new`` ([T, 512 + rope_dim] bf16) the step's latent rows are first written
    into the cache (``mla_run_append``).  ``q_pe`` may be None for a plan with
    ``rope_dim=0``."""
    import torch

    T, H, R = plan.token_capacity, plan.num_heads, plan.rope_dim
    width = KV_LORA_RANK + R
    _check_cache_shape(cache, plan.num_pages, plan.page_size, R)
    _check_dev_tensor(q_nope, "q_nope", torch.bfloat16, (T, H, KV_LORA_RANK))
    if R > 0 or q_pe is not None:
        _check_dev_tensor(q_pe, "q_pe", torch.bfloat16, (T, H, R))
    _check_dev_tensor(cache, "cache", torch.bfloat16, tuple(cache.shape))
    if out is None:
        out = torch.empty((T, H, KV_LORA_RANK), dtype=torch.bfloat16, device=q_nope.device)
    _check_dev_tensor(out, "out", torch.bfloat16, (T, H, KV_LORA_RANK))
    if return_lse and lse is None:
        lse = torch.empty((T, H), dtype=torch.float32, device=q_nope.device)
    if lse is not None:
        _check_dev_tensor(lse, "lse", torch.float32, (T, H))
    if kv_new is not None:
        _check_dev_tensor(kv_new, "kv_new", torch.bfloat16, (T, width))
    if stream is None:
        stream = torch.cuda.current_stream(q_nope.device).cuda_stream
    lib = load_library()
    lse_p = ctypes.c_void_p(lse.data_ptr() if lse is not None else 0)
    qpe_p = ctypes.c_void_p(q_pe.data_ptr() if q_pe is not None else 0)
    if kv_new is None:
        st = lib.mla_run(plan.handle, ctypes.c_void_p(q_nope.data_ptr()), qpe_p,
                         ctypes.c_void_p(cache.data_ptr()), ctypes.c_void_p(out.data_ptr()), lse_p,
                         ctypes.c_void_p(stream or 0))
        what = "mla_run"
    else:
        st = lib.mla_run_append(plan.handle, ctypes.c_void_p(q_nope.data_ptr()), qpe_p,
                                ctypes.c_void_p(kv_new.data_ptr()), ctypes.c_void_p(cache.data_ptr()),
                                ctypes.c_void_p(out.data_ptr()), lse_p, ctypes.c_void_p(stream or 0))
        what = "mla_run_append"
    if st != MLA_OK:
        raise MlaError(st, what)
    return (out, lse) if (return_lse or lse is not None) else out


def mla_append_kv(plan: MlaPlan, kv_new, cache, stream=None) -> None:
    """Write the step's latent rows ``kv_new`` [T, 576] into their cache slots
    (``mla_append_kv``)."""
    import torch

    width = KV_LORA_RANK + plan.rope_dim
    _check_cache_shape(cache, plan.num_pages, plan.page_size, plan.rope_dim)
    _check_dev_tensor(kv_new, "kv_new", torch.bfloat16, (plan.token_capacity, width))
    _check_dev_tensor(cache, "cache", torch.bfloat16, tuple(cache.shape))
    if stream is None:
        stream = torch.cuda.current_stream(kv_new.device).cuda_stream
    st = load_library().mla_append_kv(plan.handle, ctypes.c_void_p(kv_new.data_ptr()),
                                      ctypes.c_void_p(cache.data_ptr()), ctypes.c_void_p(stream or 0))
    if st != MLA_OK:
        raise MlaError(st, "mla_append_kv")


def mla_merge_state(out_a, lse_a, out_b, lse_b, out=None, lse=None, stream=None):
    """Merge two attention states over disjoint key sets by their log-sum-exps
    (``mla_merge_state``).  ``out_*`` bf16 [..., 512], ``lse_*`` fp32 [...].  Returns
    ``(out, lse)``; ``out`` may be ``out_a`` or ``out_b``."""
    import torch

    shape = tuple(out_a.shape)
    if len(shape) < 1 or shape[-1] != KV_LORA_RANK:
        raise ValueError("out_a must be [..., 512]")
    _check_dev_tensor(out_a, "out_a", torch.bfloat16, shape)
    _check_dev_tensor(out_b, "out_b", torch.bfloat16, shape)
    _check_dev_tensor(lse_a, "lse_a", torch.float32, shape[:-1])
    _check_dev_tensor(lse_b, "lse_b", torch.float32, shape[:-1])
    if out is None:
        out = torch.empty_like(out_a)
    if lse is None:
        lse = torch.empty_like(lse_a)
    _check_dev_tensor(out, "out", torch.bfloat16, shape)
    _check_dev_tensor(lse, "lse", torch.float32, shape[:-1])
    if stream is None:
        stream = torch.cuda.current_stream(out_a.device).cuda_stream
    rows = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    st = load_library().mla_merge_state(
        ctypes.c_void_p(out_a.data_ptr()), ctypes.c_void_p(lse_a.data_ptr()), ctypes.c_void_p(out_b.data_ptr()),
        ctypes.c_void_p(lse_b.data_ptr()), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_int64(rows), ctypes.c_void_p(stream or 0))
    if st != MLA_OK:
        raise MlaError(st, "mla_merge_state")
    return out, lse


def mla_plan_kernel_times(plan: MlaPlan, capacity: int = 256):
    """(attn_ms, merge_ms) arrays of the plan's recent runs (plans made with
    ``debug_flags=MLA_DEBUG_KERNEL_TIMING``)."""
    a = np.zeros(max(1, capacity), dtype=np.float32)
    m = np.zeros(max(1, capacity), dtype=np.float32)
    n = ctypes.c_int32(0)
    st = load_library().mla_plan_kernel_times(plan.handle, capacity, a.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                                              m.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), ctypes.byref(n))
    if st != MLA_OK:
        raise MlaError(st, "mla_plan_kernel_times")
    return a[: n.value], m[: n.value]


def mla_run_noalloc(qo_indptr, kv_indptr, kv_indices, last_page_len, q_nope, q_pe, cache, out, lse=None, *,
                    num_heads: int, page_size: int, num_pages: int, sm_scale: float, causal: bool = True,
                    kv_lora_rank: int = KV_LORA_RANK, rope_dim: int = ROPE_DIM, stream=None, status=None) -> None:
    """Plan and run one step without allocating (``mla_run_noalloc``): for callers that
    may not allocate device memory when attention runs.  ``out`` (and ``lse`` if given)
    must be preallocated by the caller; host tables as for ``mla_plan``.  ``status``
    (optional, a preallocated int32 CUDA tensor of one element) receives the step's
    device status once the stream has passed it (0, or MLA_ERR_DEVICE_TIMEOUT in the low
    byte).  Calls share one fixed device scratch array, so they must not overlap, and
    cannot be captured into a CUDA graph."""
    import torch

    _check_cache_shape(cache, num_pages, page_size, rope_dim)

    qo = _i32(qo_indptr)
    kvp = _i32(kv_indptr)
    kvi = _i32(kv_indices)
    last = _i32(last_page_len)
    batch = len(qo) - 1
    if batch < 0 or len(kvp) != batch + 1 or len(last) != batch or len(kvi) < int(kvp[-1]):
        raise MlaError(MLA_ERR_INVALID_ARGUMENT, "mla_run_noalloc: table lengths")
    T = int(qo[-1])
    _check_dev_tensor(q_nope, "q_nope", torch.bfloat16, (T, num_heads, kv_lora_rank))
    if rope_dim > 0 or q_pe is not None:
        _check_dev_tensor(q_pe, "q_pe", torch.bfloat16, (T, num_heads, rope_dim))
    _check_dev_tensor(cache, "cache", torch.bfloat16, tuple(cache.shape))
    _check_dev_tensor(out, "out", torch.bfloat16, (T, num_heads, kv_lora_rank))
    if lse is not None:
        _check_dev_tensor(lse, "lse", torch.float32, (T, num_heads))
    if status is not None:
        _check_dev_tensor(status, "status", torch.int32, (1,))
    if stream is None:
        stream = torch.cuda.current_stream(q_nope.device).cuda_stream
    dims = _Dims(num_heads, kv_lora_rank, rope_dim, page_size, num_pages, sm_scale)
    kvi_arr = kvi if len(kvi) else np.zeros(1, dtype=np.int32)
    st = load_library().mla_run_noalloc(
        ctypes.byref(dims), batch, _ptr(qo), _ptr(kvp), _ptr(kvi_arr), _ptr(last), 1 if causal else 0,
        ctypes.c_void_p(q_nope.data_ptr()), ctypes.c_void_p(q_pe.data_ptr() if q_pe is not None else 0),
        ctypes.c_void_p(cache.data_ptr()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr() if lse is not None else 0),
        ctypes.c_void_p(stream or 0), ctypes.c_void_p(status.data_ptr() if status is not None else 0))
    if st != MLA_OK:
        raise MlaError(st, "mla_run_noalloc")


def mla_plan_check(plan: MlaPlan) -> int:
    """Wait for the plan's last run; return its device status (0 = ok)."""
    return int(load_library().mla_plan_check(plan.handle))


def mla_plan_destroy(plan: MlaPlan) -> None:
    plan.destroy()
