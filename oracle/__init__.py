"""CPU oracle for the LSCD SpMM path (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The product path never calls
it, and it shares no code with the CUDA library: the arithmetic lives in
``tcsl_ref.c`` (plain C, fp64 accumulation), which this module compiles with
gcc and loads through ctypes.

What it computes follows the Flash-LLM paper review page (xllm-io.github.io):
section 3 "core formulas" (C = A x B and the compute-intensity bound) and
section 3 "sparse encoding format: Tiled-CSL" (per-tile word lists of
[16-bit value | 16-bit in-tile index] plus TileOffsets).  The readings taken
where the page is silent are listed at the top of ``tcsl_ref.c``.

Parity pins: every function here is pinned by ``tests/test_oracle.py``
against hand-derived golden fixtures, a brute-force dense product, closed
forms, invariants and numpy's own fp16 rounding.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "tcsl_ref.c"
_LIB = _HERE / "libtcsl_ref.so"
_lib = None

SENTINEL = 0xFFFF0000


def build(force: bool = False) -> Path:
    """Compile the oracle (no fast-math, no FMA contraction)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.tmp{os.getpid()}")
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
                               "-shared", "-fPIC", "-pthread", str(_SRC), "-o", str(tmp), "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = configure(ctypes.CDLL(str(_LIB)))
    return _lib


def configure(lib):
    """Declare the C signatures on a loaded copy of the oracle library."""
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.ref_half_to_double.restype = ctypes.c_double
    lib.ref_half_to_double.argtypes = [ctypes.c_uint16]
    lib.ref_double_to_half.restype = ctypes.c_uint16
    lib.ref_double_to_half.argtypes = [ctypes.c_double]
    lib.ref_ci.restype = ctypes.c_double
    lib.ref_ci.argtypes = [ctypes.c_double] * 4
    lib.ref_tcsl_count.argtypes = [P, I64, I64, I64, I64, P, P]
    lib.ref_tcsl_fill.argtypes = [P, I64, I64, I64, I64, P, P]
    lib.ref_tcsl_decode.argtypes = [P, P, I64, I64, I64, I64, P]
    lib.ref_tcsl_reorder_banks.argtypes = [P, P, I64, I64, I64]
    lib.ref_spmm.argtypes = [P, P, I64, I64, I64, I64, P, I64, P, P, P, ctypes.c_int]
    lib.ref_spmm_rows.argtypes = [P, P, I64, I64, I64, I64, P, I64, P, I64, P, P]
    lib.ref_dense.argtypes = [P, P, I64, I64, I64, P]
    lib.ref_dense.restype = None
    lib.ref_half_to_double_array.argtypes = [P, P, I64]
    lib.ref_half_to_double_array.restype = None
    lib.ref_double_to_half_array.argtypes = [P, P, I64]
    lib.ref_double_to_half_array.restype = None
    for f in ("ref_tcsl_count", "ref_tcsl_fill", "ref_tcsl_decode", "ref_tcsl_reorder_banks", "ref_spmm",
              "ref_spmm_rows"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


class OracleError(RuntimeError):
    pass


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError("expected float16 or uint16 bit patterns")
    return a


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what} failed with status {rc}")


def num_tiles(M: int, K: int, tile_m: int, tile_k: int) -> int:
    return -(-M // tile_m) * -(-K // tile_k)


def tcsl_count(A, tile_m: int = 64, tile_k: int = 64):
    """Tile offsets (int32, num_tiles + 1) and nnz of the fp16 matrix A."""
    lib = _load()
    A = _bits16(A)
    M, K = A.shape
    off = np.zeros(num_tiles(M, K, tile_m, tile_k) + 1, dtype=np.int32)
    nnz = np.zeros(1, dtype=np.int64)
    _check(lib.ref_tcsl_count(_ptr(A), M, K, tile_m, tile_k, _ptr(off), _ptr(nnz)), "count")
    return off, int(nnz[0])


def tcsl_encode(A, tile_m: int = 64, tile_k: int = 64, order: int = 0):
    """Tiled-CSL encoding of A: (tile_offsets int32, words uint32, nnz).

    order 0: words of a tile in ascending loc (reading R5).  order 1: the
    bank-balanced word order v2 (64 x 64 tiles only; see ref_tcsl_reorder_banks)."""
    lib = _load()
    A = _bits16(A)
    M, K = A.shape
    off, nnz = tcsl_count(A, tile_m, tile_k)
    words = np.zeros(int(off[-1]), dtype=np.uint32)
    _check(lib.ref_tcsl_fill(_ptr(A), M, K, tile_m, tile_k, _ptr(off), _ptr(words)), "fill")
    if order == 1:
        _check(lib.ref_tcsl_reorder_banks(_ptr(off), _ptr(words), len(off) - 1, tile_m, tile_k), "reorder")
    elif order != 0:
        raise ValueError("order must be 0 (ascending loc) or 1 (bank-balanced)")
    return off, words, nnz


def bank_of_loc(loc):
    """Shared-memory bank of the value at in-tile loc in the 64 x 64 swizzled dense tile
    (the quantity the v2 word order balances)."""
    x = 2 * np.asarray(loc, dtype=np.int64)
    return ((x ^ ((x >> 3) & 0x70)) >> 2) & 31


def tcsl_decode(off, words, M: int, K: int, tile_m: int = 64, tile_k: int = 64) -> np.ndarray:
    """Dense fp16 bit patterns (uint16, M x K) from a Tiled-CSL encoding."""
    lib = _load()
    off = np.ascontiguousarray(off, dtype=np.int32)
    words = np.ascontiguousarray(words, dtype=np.uint32)
    A = np.empty((M, K), dtype=np.uint16)
    _check(lib.ref_tcsl_decode(_ptr(off), _ptr(words), M, K, tile_m, tile_k, _ptr(A)), "decode")
    return A


def spmm(off, words, M: int, K: int, B, tile_m: int = 64, tile_k: int = 64, nthreads: int = 1):
    """C = A x B over the nonzero list with fp64 accumulation.

    B is the ``[N, K]`` fp16 array (K x N column-major).  Returns
    ``(C64, absC64, C16)`` each shaped ``[N, M]`` (column-major M x N): the
    fp64 sum, the fp64 sum of |a*b| and the fp16 (RNE) rounding of C64.
    """
    lib = _load()
    off = np.ascontiguousarray(off, dtype=np.int32)
    words = np.ascontiguousarray(words, dtype=np.uint32)
    B = _bits16(B)
    N = B.shape[0]
    assert B.shape[1] == K
    C64 = np.empty((N, M), dtype=np.float64)
    absC = np.empty((N, M), dtype=np.float64)
    C16 = np.empty((N, M), dtype=np.uint16)
    _check(lib.ref_spmm(_ptr(off), _ptr(words), M, K, tile_m, tile_k, _ptr(B), N,
                        _ptr(C64), _ptr(absC), _ptr(C16), int(nthreads)), "spmm")
    return C64, absC, C16.view(np.float16)


def spmm_rows(off, words, M: int, K: int, B, rows, tile_m: int = 64, tile_k: int = 64):
    """Selected rows of C: returns (C64, absC64) shaped [len(rows), N]."""
    lib = _load()
    off = np.ascontiguousarray(off, dtype=np.int32)
    words = np.ascontiguousarray(words, dtype=np.uint32)
    B = _bits16(B)
    N = B.shape[0]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    C64 = np.empty((rows.size, N), dtype=np.float64)
    absC = np.empty((rows.size, N), dtype=np.float64)
    _check(lib.ref_spmm_rows(_ptr(off), _ptr(words), M, K, tile_m, tile_k, _ptr(B), N,
                             _ptr(rows), rows.size, _ptr(C64), _ptr(absC)), "spmm_rows")
    return C64, absC


def dense(A, B) -> np.ndarray:
    """Brute-force fp64 product over every k (zeros included); [N, M]."""
    lib = _load()
    A = _bits16(A)
    B = _bits16(B)
    M, K = A.shape
    N = B.shape[0]
    C64 = np.empty((N, M), dtype=np.float64)
    lib.ref_dense(_ptr(A), _ptr(B), M, K, N, _ptr(C64))
    return C64


def half_to_double(h) -> np.ndarray:
    lib = _load()
    h = _bits16(np.asarray(h))
    out = np.empty(h.shape, dtype=np.float64)
    lib.ref_half_to_double_array(_ptr(h), _ptr(out), h.size)
    return out


def double_to_half(x) -> np.ndarray:
    """fp16 bit patterns (uint16) of the RNE rounding of fp64 values."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib.ref_double_to_half_array(_ptr(x), _ptr(out), x.size)
    return out


def ci(M: float, K: float, N: float, sizeof_dtype: float = 2.0) -> float:
    """Compute intensity 2MNK / ((MK + KN + MN) * sizeof)."""
    return _load().ref_ci(float(M), float(K), float(N), float(sizeof_dtype))


def tolerance_ok(C, C64, absC64):
    """Element-wise parity bound |C - C64| <= 2^-10 |C64| + 1e-4 * sum|a b|.

    NaN must match NaN; equal infinities match.  Returns a boolean array.
    """
    C = np.asarray(C, dtype=np.float64)
    both_nan = np.isnan(C) & np.isnan(C64)
    same_inf = np.isinf(C) & np.isinf(C64) & (np.sign(C) == np.sign(C64))
    with np.errstate(invalid="ignore"):
        err = np.abs(C - C64)
        ok = err <= (2.0 ** -10) * np.abs(C64) + 1e-4 * absC64
    return ok | both_nan | same_inf
