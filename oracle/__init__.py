"""CPU oracle for head-aware paged attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  It shares no code with the CUDA
path (``head_aware_paged_build_b200``): its arithmetic lives in
``segpaged_oracle.c`` (fp64 dense attention with an explicit visibility mask)
and in ``brute.py`` (a pure-Python enumeration used to pin it).

Head kinds are the strings ``"global"``, ``"local"``, ``"dense"`` and
``"retrieval"``; a retrieval head also takes ``sel`` (kept blocks, from
``retrieval_select``) and ``block`` (positions per block, the page size).
Pinned functions: ``attention_rows`` / ``attention_batch`` (brute force,
causal-attention special case, closed forms), ``stored_mask`` /
``visible_pairs`` (brute-force union and closed forms), ``retrieval_select``
(brute force over block subsets, closed forms), the E4M3 encoder / decoder.
Nothing here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "segpaged_oracle.c"
_BUILD = _HERE / "_build"
_LIB_PATH = _BUILD / "libsegpaged_oracle.so"
_KIND = {"global": 0, "local": 1, "dense": 2, "retrieval": 3}

_lib = None


def build(force: bool = False, out: Path | None = None, extra_flags: tuple[str, ...] = ()) -> Path:
    """Compile the oracle with gcc (-O2 -fopenmp, no fast-math); returns the .so path."""
    out = out or _LIB_PATH
    out.parent.mkdir(parents=True, exist_ok=True)
    if force or not out.exists() or out.stat().st_mtime < _SRC.stat().st_mtime:
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               *extra_flags, str(_SRC), "-o", str(out), "-lm"]
        subprocess.run(cmd, check=True)
    return out


def _bind(lib):
    i64, dbl, p = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    lib.oracle_attention_rows.argtypes = [i64, i64, p, p, i64, p, p, ctypes.c_int, i64, i64, p, i64, dbl, p, p]
    lib.oracle_attention_rows.restype = ctypes.c_int
    lib.oracle_stored_mask.argtypes = [ctypes.c_int, i64, i64, p, i64, i64, i64, p]
    lib.oracle_stored_mask.restype = i64
    lib.oracle_visible_pairs.argtypes = [ctypes.c_int, i64, i64, p, i64, i64, i64]
    lib.oracle_visible_pairs.restype = i64
    lib.oracle_retrieval_select.argtypes = [i64, i64, i64, ctypes.c_float, p, p]
    lib.oracle_retrieval_select.restype = i64
    lib.oracle_attention_batch.argtypes = [i64, i64, p, p, p, i64, p, p, p, p, p, p, p, p, dbl, p, p]
    lib.oracle_attention_batch.restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_e4m3_encode.argtypes = [i64, p, ctypes.c_float, p]
    lib.oracle_e4m3_encode.restype = None
    lib.oracle_e4m3_decode.argtypes = [i64, p, dbl, p]
    lib.oracle_e4m3_decode.restype = None
    lib.oracle_block_mass.argtypes = [i64, i64, p, i64, p, dbl, i64, p]
    lib.oracle_block_mass.restype = ctypes.c_int
    return lib


def load(path: Path | None = None):
    """Load (building if needed) the oracle library.  A path loads a variant build."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(str(path)))
    if _lib is None:
        # A planted-mistake build of the oracle (tests/test_oracle_mutants.py) is
        # selected through this variable; normal runs never set it.
        override = os.environ.get("SEGPAGED_ORACLE_LIB")
        _lib = _bind(ctypes.CDLL(override if override else str(build())))
    return _lib


def num_threads() -> int:
    return int(load().oracle_num_threads())


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _sel(kind: str, sel, block: int, L: int):
    """Kept-block array of a retrieval head (uint8), or None for other kinds."""
    if kind != "retrieval":
        return None
    if sel is None or block < 1:
        raise ValueError("oracle: a retrieval head needs its kept blocks (sel) and the block size")
    a = np.ascontiguousarray(np.asarray(sel, dtype=np.uint8))
    if a.size < -(-L // block):
        raise ValueError("oracle: sel has fewer entries than the context has blocks")
    return a


def _sel_ptr(a):
    return _ptr(a) if a is not None else None


def attention_rows(q, pos, k, v, kind: str, sink: int, window: int, scale: float | None = None,
                   lib=None, sel=None, block: int = 0):
    """fp64 attention of query rows ``q [n, d]`` at positions ``pos [n]`` over dense ``k, v [L, d]``.

    Returns ``(out [n, d], lse [n])`` in fp64.  ``scale`` defaults to 1/sqrt(d).  A retrieval
    head needs ``sel`` (kept blocks) and ``block`` (positions per block).
    """
    lib = lib or load()
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    n, d = q.shape
    L = k.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(np.float64(d))
    sa = _sel(kind, sel, block, L)
    out = np.empty((n, d), np.float64)
    lse = np.empty(n, np.float64)
    rc = lib.oracle_attention_rows(n, d, _ptr(q), _ptr(pos), L, _ptr(k), _ptr(v), _KIND[kind],
                                   int(sink), int(window), _sel_ptr(sa), int(block), float(scale), _ptr(out),
                                   _ptr(lse))
    if rc != 0:
        raise ValueError("oracle: a query position lies outside the context or sees nothing")
    return out, lse


def attention_batch(groups, scale: float | None = None, lib=None):
    """fp64 attention of the rows of many (sequence, kv-head) groups in one parallel loop.

    ``groups`` is a sequence of ``(q [n_g, d], pos [n_g], k [L_g, d], v [L_g, d], kind, sink, window)``,
    with ``sel, block`` appended for a retrieval head.
    Each row is computed exactly as by ``attention_rows``; every host core works on
    the batch's rows together.  Returns a list of ``(out [n_g, d], lse [n_g])`` per group.
    """
    lib = lib or load()
    if not groups:
        return []
    d = int(np.asarray(groups[0][0]).shape[1])
    qs, poss, gid, ks, vs = [], [], [], [], []
    Ls, kinds, sinks, wins, sels, blocks = [], [], [], [], [], []
    for g, grp in enumerate(groups):
        q, pos, k, v, kind, sink, window = grp[:7]
        sel, block = (grp[7], grp[8]) if len(grp) > 7 else (None, 0)
        q = np.ascontiguousarray(q, dtype=np.float64)
        qs.append(q)
        poss.append(np.asarray(pos, np.int64))
        gid.append(np.full(q.shape[0], g, np.int64))
        ks.append(np.ascontiguousarray(k, dtype=np.float64))
        vs.append(np.ascontiguousarray(v, dtype=np.float64))
        Ls.append(ks[-1].shape[0])
        kinds.append(_KIND[kind])
        sinks.append(int(sink))
        wins.append(int(window))
        sels.append(_sel(kind, sel, int(block), ks[-1].shape[0]))
        blocks.append(int(block))
    q = np.ascontiguousarray(np.concatenate(qs, 0))
    pos = np.ascontiguousarray(np.concatenate(poss))
    gid = np.ascontiguousarray(np.concatenate(gid))
    n = q.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(np.float64(d))
    kp = (ctypes.c_void_p * len(groups))(*[a.ctypes.data for a in ks])
    vp = (ctypes.c_void_p * len(groups))(*[a.ctypes.data for a in vs])
    L = np.asarray(Ls, np.int64)
    kind_a = np.asarray(kinds, np.int32)
    sink_a = np.asarray(sinks, np.int64)
    win_a = np.asarray(wins, np.int64)
    sp = (ctypes.c_void_p * len(groups))(*[a.ctypes.data if a is not None else None for a in sels])
    blk_a = np.asarray(blocks, np.int64)
    out = np.empty((n, d), np.float64)
    lse = np.empty(n, np.float64)
    rc = lib.oracle_attention_batch(n, d, _ptr(q), _ptr(pos), _ptr(gid), len(groups), _ptr(L), kp, vp,
                                    _ptr(kind_a), _ptr(sink_a), _ptr(win_a), sp, _ptr(blk_a), float(scale),
                                    _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle: a query position lies outside the context or sees nothing")
    res, r0 = [], 0
    for qq in qs:
        res.append((out[r0:r0 + qq.shape[0]], lse[r0:r0 + qq.shape[0]]))
        r0 += qq.shape[0]
    return res


def stored_mask(kind: str, sink: int, window: int, L: int, q0: int, lib=None, sel=None,
                block: int = 0) -> np.ndarray:
    """Positions of [0, L) a head must keep for queries at q0 .. L-1 (bool [L])."""
    lib = lib or load()
    sa = _sel(kind, sel, block, L)
    m = np.zeros(L, np.uint8)
    lib.oracle_stored_mask(_KIND[kind], int(sink), int(window), _sel_ptr(sa), int(block), int(L), int(q0), _ptr(m))
    return m.astype(bool)


def visible_pairs(kind: str, sink: int, window: int, L: int, q0: int, lib=None, sel=None, block: int = 0) -> int:
    """Number of (query, key) pairs evaluated for queries at q0 .. L-1."""
    lib = lib or load()
    sa = _sel(kind, sel, block, L)
    return int(lib.oracle_visible_pairs(_KIND[kind], int(sink), int(window), _sel_ptr(sa), int(block), int(L),
                                        int(q0)))


def retrieval_select(L: int, block: int, sink: int, top_p: float, mass, lib=None) -> np.ndarray:
    """Kept blocks of a retrieval head (bool [ceil(L / block)]) from its per-block importance ``mass``.

    The smallest set of candidate blocks (blocks holding a position >= sink), in decreasing
    order of importance (ties: lower block first), whose importance reaches the fraction
    ``top_p`` (as float32) of the candidates' total; sums in fp64 in that order; top_p >= 1
    keeps every candidate, top_p <= 0 none.
    """
    lib = lib or load()
    n = -(-int(L) // int(block))
    m = np.ascontiguousarray(np.asarray(mass, dtype=np.float32))
    if m.size != n:
        raise ValueError(f"oracle: {n} block masses expected, got {m.size}")
    sel = np.zeros(n, np.uint8)
    if lib.oracle_retrieval_select(int(L), int(block), int(sink), float(np.float32(top_p)), _ptr(m), _ptr(sel)) < 0:
        raise ValueError("oracle: block masses must be finite and non-negative")
    return sel.astype(bool)


def problem_rows(q_rows, q_positions, k_dense, v_dense, kind, sink, window, scale=None, lib=None, sel=None,
                 block: int = 0):
    """Same as attention_rows; accepts torch tensors (any float dtype, upcast exactly)."""
    def np64(t):
        if hasattr(t, "detach"):
            return t.detach().to("cpu").double().numpy()
        return np.asarray(t, np.float64)
    return attention_rows(np64(q_rows), np.asarray(q_positions, np.int64), np64(k_dense),
                          np64(v_dense), kind, sink, window, scale, lib, sel=sel, block=block)


def e4m3_encode(x, inv_scale: float, lib=None) -> np.ndarray:
    """E4M3 codes (uint8) of fp32(x * inv_scale): nearest, ties to even, saturating at +-448."""
    lib = lib or load()
    xf = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    codes = np.empty(xf.shape, np.uint8)
    lib.oracle_e4m3_encode(xf.size, _ptr(xf), float(np.float32(inv_scale)), _ptr(codes))
    return codes


def e4m3_decode(codes, scale: float, lib=None) -> np.ndarray:
    """fp64 values of E4M3 codes times scale."""
    lib = lib or load()
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    out = np.empty(c.shape, np.float64)
    lib.oracle_e4m3_decode(c.size, _ptr(c), float(scale), _ptr(out))
    return out


def block_mass(q, k, block: int, scale: float | None = None, lib=None) -> np.ndarray:
    """Attention mass per block of ``block`` positions (fp64, [ceil(L / block)]).

    ``q [g, d]``: the g queries of one kv-head's group at the last position of the
    context; ``k [L, d]``: the context's keys.  Each query's softmax over all L
    positions, summed per block and averaged over the g queries (the importance a
    retrieval head's top-p selection reads).  ``scale`` defaults to 1/sqrt(d).
    """
    lib = lib or load()
    q = np.ascontiguousarray(np.atleast_2d(q), dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    g, d = q.shape
    L = k.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(np.float64(d))
    out = np.empty(-(-L // int(block)), np.float64)
    if lib.oracle_block_mass(g, d, _ptr(q), L, _ptr(k), float(scale), int(block), _ptr(out)) != 0:
        raise ValueError("oracle: block_mass needs g, d, L, block >= 1")
    return out
