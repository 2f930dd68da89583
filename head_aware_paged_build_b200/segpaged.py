"""Python binding of libsegpaged.so (ctypes; argument marshalling only).

Every function here has the name of a C entry point in ``include/segpaged.h``
and forwards to it; no step of the attention path runs in Python.  Device
buffers are passed as raw pointers (``int`` addresses, e.g. ``tensor.data_ptr()``)
and streams as ``cudaStream_t`` handles (``torch.cuda.Stream.cuda_stream``).

Loading fails loudly when the compiled library is missing: there is no CPU
or library fallback.
"""
from __future__ import annotations

import ctypes
from pathlib import Path
from typing import Sequence

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libsegpaged.so"

SP_OK, SP_ERR_INVALID_ARG, SP_ERR_UNSUPPORTED, SP_ERR_WORKSPACE, SP_ERR_CUDA, SP_ERR_DEVICE_CHECK = range(6)
SP_GLOBAL, SP_LOCAL, SP_DENSE, SP_RETRIEVAL = range(4)
SP_F32, SP_BF16, SP_E4M3 = 0, 1, 2
SP_FLAG_DENSE_MASKED = 1
SP_FLAG_RING = 2
SP_VARLEN = -1
KIND_CODES = {"global": SP_GLOBAL, "local": SP_LOCAL, "dense": SP_DENSE, "retrieval": SP_RETRIEVAL}
DTYPE_CODES = {"f32": SP_F32, "bf16": SP_BF16, "e4m3": SP_E4M3}

# every symbol include/segpaged.h declares
EXPORTED = ("segpaged_plan_create", "segpaged_plan_destroy", "segpaged_plan_sizes",
            "segpaged_plan_head_segments", "segpaged_plan_head_pages", "segpaged_plan_decode_items",
            "segpaged_plan_prefill_items", "segpaged_table_write",
            "build_segpaged_cache", "build_segpaged_cache_layers", "segpaged_gather", "segpaged_attention",
            "segpaged_attention_decode_noalloc", "segpaged_decode_append", "segpaged_decode_step",
            "segpaged_read_device_status",
            "segpaged_clear_device_status", "segpaged_eval_exp2_fma", "segpaged_block_mass_workspace",
            "segpaged_block_mass", "segpaged_status_string", "segpaged_last_error", "segpaged_abi_version")


class SegPagedError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {status_name(status)}: {detail}")


class sp_head_policy(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("sink", ctypes.c_int32), ("window", ctypes.c_int32),
                ("top_p", ctypes.c_float)]


class sp_problem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("ctx_len", ctypes.POINTER(ctypes.c_int32)), ("q_start", ctypes.POINTER(ctypes.c_int32)),
                ("policy", ctypes.POINTER(sp_head_policy)), ("first_page", ctypes.c_int64),
                ("page_ids", ctypes.POINTER(ctypes.c_int32)), ("target_ctas", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("append_capacity", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float),
                ("block_mass", ctypes.POINTER(ctypes.POINTER(ctypes.c_float))), ("spare_pages", ctypes.c_int32)]


class sp_sizes(ctypes.Structure):
    _fields_ = [("num_pages", ctypes.c_int64), ("pool_pages", ctypes.c_int64), ("page_bytes", ctypes.c_int64),
                ("table_bytes", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64),
                ("stored_token_heads", ctypes.c_int64), ("dense_token_heads", ctypes.c_int64),
                ("visible_pairs", ctypes.c_int64), ("num_queries", ctypes.c_int64), ("is_decode", ctypes.c_int32),
                ("num_decode_ctas", ctypes.c_int32), ("num_prefill_items", ctypes.c_int32),
                ("num_combine", ctypes.c_int32), ("launches_per_call", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}

    def kernel_launches(self) -> int:
        """Kernels one segpaged_attention call launches."""
        return int(self.launches_per_call)


class sp_segment(ctypes.Structure):
    _fields_ = [("abs_start", ctypes.c_int32), ("length", ctypes.c_int32), ("first_page_index", ctypes.c_int32),
                ("num_pages", ctypes.c_int32)]


_lib = None


def load(path: Path | str | None = None) -> ctypes.CDLL:
    """Load libsegpaged.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = Path(path) if path else LIB_PATH
    if not p.exists():
        raise ImportError(f"{p} is missing: build it with head_aware_paged_build_b200.build_ext.build() "
                          "(there is no fallback path)")
    lib = ctypes.CDLL(str(p))
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "segpaged_plan_create": ([ctypes.POINTER(sp_problem), ctypes.POINTER(vp)], i32),
        "segpaged_plan_destroy": ([vp], None),
        "segpaged_plan_sizes": ([vp, ctypes.POINTER(sp_sizes)], i32),
        "segpaged_plan_head_segments": ([vp, i32, i32, ctypes.POINTER(sp_segment), i32, ctypes.POINTER(i32)], i32),
        "segpaged_plan_head_pages": ([vp, i32, i32, ctypes.POINTER(i64), i32, ctypes.POINTER(i32)], i32),
        "segpaged_plan_decode_items": ([vp, ctypes.POINTER(i32), i32, ctypes.POINTER(i32)], i32),
        "segpaged_plan_prefill_items": ([vp, ctypes.POINTER(i32), i32, ctypes.POINTER(i32)], i32),
        "segpaged_table_write": ([vp, vp, sz, vp], i32),
        "build_segpaged_cache": ([vp, vp, vp, vp, i64, i64, i64, vp, vp, vp], i32),
        "build_segpaged_cache_layers": ([i32, ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                                         ctypes.POINTER(vp), i64, i64, i64, vp, vp, vp], i32),
        "segpaged_gather": ([vp, vp, vp, vp, vp, vp, i64, i64, i64, vp], i32),
        "segpaged_attention": ([vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, sz, vp], i32),
        "segpaged_attention_decode_noalloc": ([vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp], i32),
        "segpaged_decode_append": ([vp, vp, vp, vp, i64, i64, vp, vp, vp, vp], i32),
        "segpaged_decode_step": ([vp, vp, vp, vp, i64, i64, vp, vp, vp, vp, vp, ctypes.c_float, vp, sz, vp], i32),
        "segpaged_read_device_status": ([vp, ctypes.POINTER(i32), vp], i32),
        "segpaged_clear_device_status": ([vp, vp], i32),
        "segpaged_eval_exp2_fma": ([vp, vp, i64, vp], i32),
        "segpaged_block_mass_workspace": ([ctypes.POINTER(sp_problem), ctypes.POINTER(sz)], i32),
        "segpaged_block_mass": ([ctypes.POINTER(sp_problem), vp, i64, i64, i64, vp, ctypes.c_float, vp, i64, vp,
                                 sz, vp], i32),
        "segpaged_status_string": ([i32], ctypes.c_char_p),
        "segpaged_last_error": ([], ctypes.c_char_p),
        "segpaged_abi_version": ([], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    if path is None:
        _lib = lib
    return lib


def status_name(st: int) -> str:
    return load().segpaged_status_string(st).decode()


def last_error() -> str:
    return load().segpaged_last_error().decode()


def _check(st: int, where: str) -> None:
    if st != SP_OK:
        raise SegPagedError(st, where, last_error())


# ---------------------------------------------------------------------------
# Thin wrappers with the C names
# ---------------------------------------------------------------------------

def make_problem(batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int, page_size: int, dtype: str,
                 ctx_len: Sequence[int], q_start: Sequence[int], policy: Sequence[tuple],
                 first_page: int = 0, page_ids: Sequence[int] | None = None, target_ctas: int = 0,
                 flags: int = 0, append_capacity: int = 0, kv_dtype: str | int | None = None,
                 k_scale: float = 1.0, v_scale: float = 1.0, block_mass: Sequence | None = None,
                 spare_pages: int = 0):
    """Build an ``sp_problem`` plus the host arrays it points to (kept alive in the result).

    ``policy`` entries are ``(kind, sink, window)`` or, for retrieval heads,
    ``(kind, sink, window, top_p)``; ``block_mass`` is None or one entry per
    (sequence, kv-head): the importance of each page-size block (a float
    sequence) for a retrieval head, None for the others.
    """
    B = batch
    ctx = (ctypes.c_int32 * B)(*ctx_len)
    q0 = (ctypes.c_int32 * B)(*q_start)
    pol = (sp_head_policy * len(policy))(*[
        sp_head_policy(KIND_CODES[e[0]] if isinstance(e[0], str) else e[0], e[1], e[2],
                       float(e[3]) if len(e) > 3 else 0.0) for e in policy])
    ids = (ctypes.c_int32 * len(page_ids))(*page_ids) if page_ids is not None else None
    masses, mass_ptrs = [], None
    if block_mass is not None:
        fp = ctypes.POINTER(ctypes.c_float)
        ptrs = []
        for m in block_mass:
            if m is None:
                ptrs.append(fp())
            else:
                arr = (ctypes.c_float * max(1, len(m)))(*[float(x) for x in m])
                masses.append(arr)
                ptrs.append(ctypes.cast(arr, fp))
        mass_ptrs = (fp * len(ptrs))(*ptrs)
    prob = sp_problem(B, num_q_heads, num_kv_heads, head_dim, page_size,
                      DTYPE_CODES[dtype] if isinstance(dtype, str) else dtype,
                      ctx, q0, pol, first_page,
                      ctypes.cast(ids, ctypes.POINTER(ctypes.c_int32)) if ids is not None else None,
                      target_ctas, flags, append_capacity,
                      0 if kv_dtype is None else (DTYPE_CODES[kv_dtype] if isinstance(kv_dtype, str) else kv_dtype),
                      k_scale, v_scale,
                      ctypes.cast(mass_ptrs, ctypes.POINTER(ctypes.POINTER(ctypes.c_float)))
                      if mass_ptrs is not None else None, spare_pages)
    prob._keep = (ctx, q0, pol, ids, masses, mass_ptrs)
    return prob


def segpaged_plan_create(problem: sp_problem) -> int:
    out = ctypes.c_void_p()
    _check(load().segpaged_plan_create(ctypes.byref(problem), ctypes.byref(out)), "segpaged_plan_create")
    return out.value


def segpaged_plan_create_status(problem: sp_problem) -> tuple[int, int | None]:
    """Like segpaged_plan_create but returns (status, plan) instead of raising."""
    out = ctypes.c_void_p()
    st = load().segpaged_plan_create(ctypes.byref(problem), ctypes.byref(out))
    return st, out.value


def segpaged_plan_destroy(plan: int) -> None:
    load().segpaged_plan_destroy(plan)


def segpaged_plan_sizes(plan: int) -> sp_sizes:
    z = sp_sizes()
    _check(load().segpaged_plan_sizes(plan, ctypes.byref(z)), "segpaged_plan_sizes")
    return z


def segpaged_plan_head_segments(plan: int, b: int, kv: int) -> list[tuple[int, int, int, int]]:
    n = ctypes.c_int32()
    _check(load().segpaged_plan_head_segments(plan, b, kv, None, 0, ctypes.byref(n)), "segpaged_plan_head_segments")
    segs = (sp_segment * max(1, n.value))()
    _check(load().segpaged_plan_head_segments(plan, b, kv, segs, n.value, ctypes.byref(n)),
           "segpaged_plan_head_segments")
    return [(s.abs_start, s.length, s.first_page_index, s.num_pages) for s in segs[: n.value]]


def segpaged_plan_head_pages(plan: int, b: int, kv: int) -> list[int]:
    n = ctypes.c_int32()
    _check(load().segpaged_plan_head_pages(plan, b, kv, None, 0, ctypes.byref(n)), "segpaged_plan_head_pages")
    ids = (ctypes.c_int64 * max(1, n.value))()
    _check(load().segpaged_plan_head_pages(plan, b, kv, ids, n.value, ctypes.byref(n)), "segpaged_plan_head_pages")
    return list(ids[: n.value])


SP_DECODE_ITEM_WORDS = 12
DECODE_ITEM_FIELDS = ("cta", "b", "kv", "page_begin", "page_end", "slot", "n_slots", "slot0", "group_size",
                      "group_slot0", "counter", "group_counter")


def segpaged_plan_decode_items(plan: int) -> list[dict]:
    """The decode work split of a plan, one dict per work item in launch order."""
    n = ctypes.c_int32()
    _check(load().segpaged_plan_decode_items(plan, None, 0, ctypes.byref(n)), "segpaged_plan_decode_items")
    rec = (ctypes.c_int32 * max(1, n.value * SP_DECODE_ITEM_WORDS))()
    _check(load().segpaged_plan_decode_items(plan, rec, n.value, ctypes.byref(n)), "segpaged_plan_decode_items")
    w = SP_DECODE_ITEM_WORDS
    return [dict(zip(DECODE_ITEM_FIELDS, rec[i * w:(i + 1) * w])) for i in range(n.value)]


SP_PREFILL_ITEM_WORDS = 16
PREFILL_ITEM_FIELDS = ("b", "kv", "tile", "qh0", "qh1", "q_row0", "q_row1", "n_rows0", "n_rows1", "p0_0", "p0_1",
                       "t0", "t1", "t2", "t3", "work")


def segpaged_plan_prefill_items(plan: int) -> list[dict]:
    """The prefill work list of a plan, one dict per item (one CTA) in launch order."""
    n = ctypes.c_int32()
    _check(load().segpaged_plan_prefill_items(plan, None, 0, ctypes.byref(n)), "segpaged_plan_prefill_items")
    rec = (ctypes.c_int32 * max(1, n.value * SP_PREFILL_ITEM_WORDS))()
    _check(load().segpaged_plan_prefill_items(plan, rec, n.value, ctypes.byref(n)), "segpaged_plan_prefill_items")
    w = SP_PREFILL_ITEM_WORDS
    return [dict(zip(PREFILL_ITEM_FIELDS, rec[i * w:(i + 1) * w])) for i in range(n.value)]


def segpaged_table_write(plan: int, d_table: int, nbytes: int, stream: int = 0) -> None:
    _check(load().segpaged_table_write(plan, d_table, nbytes, stream), "segpaged_table_write")


def build_segpaged_cache(plan: int, d_table: int, k_dense: int, v_dense: int, stride_seq: int, stride_head: int,
                         stride_tok: int, k_pool: int, v_pool: int, stream: int = 0) -> None:
    _check(load().build_segpaged_cache(plan, d_table, k_dense, v_dense, stride_seq, stride_head, stride_tok,
                                       k_pool, v_pool, stream), "build_segpaged_cache")


def build_segpaged_cache_layers(plans: Sequence[int], d_tables: Sequence[int], k_dense: Sequence[int],
                                v_dense: Sequence[int], stride_seq: int, stride_head: int, stride_tok: int,
                                k_pool: int, v_pool: int, stream: int = 0) -> None:
    n = len(plans)
    arr = lambda xs: (ctypes.c_void_p * max(1, n))(*xs)
    _check(load().build_segpaged_cache_layers(n, arr(plans), arr(d_tables), arr(k_dense), arr(v_dense), stride_seq,
                                              stride_head, stride_tok, k_pool, v_pool, stream),
           "build_segpaged_cache_layers")


def segpaged_gather(plan: int, d_table: int, k_pool: int, v_pool: int, k_out: int, v_out: int, stride_seq: int,
                    stride_head: int, stride_tok: int, stream: int = 0) -> None:
    _check(load().segpaged_gather(plan, d_table, k_pool, v_pool, k_out, v_out, stride_seq, stride_head,
                                  stride_tok, stream), "segpaged_gather")


def segpaged_attention(plan: int, d_table: int, k_pool: int, v_pool: int, q: int, out: int, lse: int | None,
                       softmax_scale: float, workspace: int, workspace_bytes: int, stream: int = 0) -> None:
    _check(load().segpaged_attention(plan, d_table, k_pool, v_pool, q, out, lse, softmax_scale, workspace,
                                     workspace_bytes, stream), "segpaged_attention")


def segpaged_attention_decode_noalloc(plan: int, d_table: int, k_pool: int, v_pool: int, q: int, out: int,
                                      lse: int | None, softmax_scale: float, d_status: int,
                                      stream: int = 0) -> None:
    """Decode attention with the library's built-in scratch (no workspace argument, no allocation).

    ``d_status`` is the caller's device int32 that receives the device status code."""
    _check(load().segpaged_attention_decode_noalloc(plan, d_table, k_pool, v_pool, q, out, lse, softmax_scale,
                                                    d_status, stream), "segpaged_attention_decode_noalloc")


def segpaged_decode_append(plan: int, d_table: int, k_new: int, v_new: int, stride_seq: int, stride_head: int,
                           k_pool: int, v_pool: int, workspace: int, stream: int = 0) -> None:
    """Append one token per sequence to a ring plan's cache, in place (device table updated)."""
    _check(load().segpaged_decode_append(plan, d_table, k_new, v_new, stride_seq, stride_head, k_pool, v_pool,
                                         workspace, stream), "segpaged_decode_append")


def segpaged_decode_step(plan: int, d_table: int, k_new: int, v_new: int, stride_seq: int, stride_head: int,
                         k_pool: int, v_pool: int, q: int, out: int, lse: int | None, softmax_scale: float,
                         workspace: int, workspace_bytes: int, stream: int = 0) -> None:
    """Append one token per sequence to a ring plan's cache and attend with it (one launch on bf16 pages)."""
    _check(load().segpaged_decode_step(plan, d_table, k_new, v_new, stride_seq, stride_head, k_pool, v_pool, q, out,
                                       lse, softmax_scale, workspace, workspace_bytes, stream), "segpaged_decode_step")


def segpaged_attention_status(*args) -> int:
    """Like segpaged_attention but returns the status code instead of raising."""
    return load().segpaged_attention(*args)


def segpaged_read_device_status(workspace: int, stream: int = 0) -> int:
    code = ctypes.c_int32()
    st = load().segpaged_read_device_status(workspace, ctypes.byref(code), stream)
    if st not in (SP_OK, SP_ERR_DEVICE_CHECK):
        _check(st, "segpaged_read_device_status")
    return code.value


def segpaged_clear_device_status(workspace: int, stream: int = 0) -> None:
    _check(load().segpaged_clear_device_status(workspace, stream), "segpaged_clear_device_status")


def segpaged_eval_exp2_fma(d_x: int, d_y: int, n: int, stream: int = 0) -> None:
    """y = the prefill kernel's FMA-pipe 2^x of x (device float arrays of n elements)."""
    _check(load().segpaged_eval_exp2_fma(d_x, d_y, n, stream), "segpaged_eval_exp2_fma")


def segpaged_block_mass_workspace(problem: sp_problem) -> int:
    """Workspace bytes segpaged_block_mass needs for ``problem``."""
    n = ctypes.c_size_t()
    _check(load().segpaged_block_mass_workspace(ctypes.byref(problem), ctypes.byref(n)),
           "segpaged_block_mass_workspace")
    return n.value


def segpaged_block_mass(problem: sp_problem, k_dense: int, stride_seq: int, stride_head: int, stride_tok: int,
                        q: int, softmax_scale: float, mass: int, mass_stride: int, workspace: int,
                        workspace_bytes: int, stream: int = 0) -> None:
    """The attention mass per page-size block of each (sequence, kv-head): a retrieval head's importance."""
    _check(load().segpaged_block_mass(ctypes.byref(problem), k_dense, stride_seq, stride_head, stride_tok, q,
                                      softmax_scale, mass, mass_stride, workspace, workspace_bytes, stream),
           "segpaged_block_mass")


def segpaged_block_mass_status(problem: sp_problem, *args) -> int:
    """Like segpaged_block_mass but returns the status code instead of raising."""
    return load().segpaged_block_mass(ctypes.byref(problem), *args)


def segpaged_abi_version() -> int:
    return load().segpaged_abi_version()
