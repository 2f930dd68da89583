"""CPU oracle for head-aware paged attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  It shares no code with the CUDA
path (``head_aware_paged_build_b200``): its arithmetic lives in
``segpaged_oracle.c`` (fp64 dense attention with an explicit visibility mask)
and in ``brute.py`` (a pure-Python enumeration used to pin it).

Head kinds are the strings ``"global"``, ``"local"`` and ``"dense"``.
Pinned functions: ``attention_rows`` (brute force, causal-attention special
case, closed forms), ``stored_mask`` / ``visible_pairs`` (brute-force union and
closed forms).  Nothing here is "parity unpinned".
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
_KIND = {"global": 0, "local": 1, "dense": 2}

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
    lib.oracle_attention_rows.argtypes = [i64, i64, p, p, i64, p, p, ctypes.c_int, i64, i64, dbl, p, p]
    lib.oracle_attention_rows.restype = ctypes.c_int
    lib.oracle_stored_mask.argtypes = [ctypes.c_int, i64, i64, i64, i64, p]
    lib.oracle_stored_mask.restype = i64
    lib.oracle_visible_pairs.argtypes = [ctypes.c_int, i64, i64, i64, i64]
    lib.oracle_visible_pairs.restype = i64
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_e4m3_encode.argtypes = [i64, p, ctypes.c_float, p]
    lib.oracle_e4m3_encode.restype = None
    lib.oracle_e4m3_decode.argtypes = [i64, p, dbl, p]
    lib.oracle_e4m3_decode.restype = None
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


def attention_rows(q, pos, k, v, kind: str, sink: int, window: int, scale: float | None = None,
                   lib=None):
    """fp64 attention of query rows ``q [n, d]`` at positions ``pos [n]`` over dense ``k, v [L, d]``.

    Returns ``(out [n, d], lse [n])`` in fp64.  ``scale`` defaults to 1/sqrt(d).
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
    out = np.empty((n, d), np.float64)
    lse = np.empty(n, np.float64)
    rc = lib.oracle_attention_rows(n, d, _ptr(q), _ptr(pos), L, _ptr(k), _ptr(v), _KIND[kind],
                                   int(sink), int(window), float(scale), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle: a query position lies outside the context or sees nothing")
    return out, lse


def stored_mask(kind: str, sink: int, window: int, L: int, q0: int, lib=None) -> np.ndarray:
    """Positions of [0, L) a head must keep for queries at q0 .. L-1 (bool [L])."""
    lib = lib or load()
    m = np.zeros(L, np.uint8)
    lib.oracle_stored_mask(_KIND[kind], int(sink), int(window), int(L), int(q0), _ptr(m))
    return m.astype(bool)


def visible_pairs(kind: str, sink: int, window: int, L: int, q0: int, lib=None) -> int:
    """Number of (query, key) pairs evaluated for queries at q0 .. L-1."""
    lib = lib or load()
    return int(lib.oracle_visible_pairs(_KIND[kind], int(sink), int(window), int(L), int(q0)))


def problem_rows(q_rows, q_positions, k_dense, v_dense, kind, sink, window, scale=None, lib=None):
    """Same as attention_rows; accepts torch tensors (any float dtype, upcast exactly)."""
    def np64(t):
        if hasattr(t, "detach"):
            return t.detach().to("cpu").double().numpy()
        return np.asarray(t, np.float64)
    return attention_rows(np64(q_rows), np.asarray(q_positions, np.int64), np64(k_dense),
                          np64(v_dense), kind, sink, window, scale, lib)


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
