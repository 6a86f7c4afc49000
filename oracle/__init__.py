"""CPU oracle for the hashed n-gram (PLE / Engram) lookup -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never loads it and
has no fallback to it.  The arithmetic lives in ``ple_oracle.cpp`` (plain
scalar C++, built with ``-O2 -ffp-contract=off``); this module only builds it
and marshals numpy arrays into it.

Pins (tests that hold the oracle to something other than itself) are in
``tests/test_oracle_pins.py``; every function below has at least one.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "ple_oracle.cpp")
LIB_PATH = os.path.join(_HERE, "libple_oracle.so")
CHUNK = 32
_lib = None

_i64p = ctypes.POINTER(ctypes.c_int64)
_i32p = ctypes.POINTER(ctypes.c_int32)
_f32p = ctypes.POINTER(ctypes.c_float)


def build(force: bool = False, sanitize: bool = False) -> str:
    """Compile the oracle with g++ (optionally an ASan/UBSan variant)."""
    out = LIB_PATH if not sanitize else os.path.join(_HERE, "libple_oracle_san.so")
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
        return out
    cmd = ["g++", "-O2", "-ffp-contract=off", "-std=c++17", "-Wall", "-Wextra", "-shared", "-fPIC",
           "-pthread", "-o", out, SRC]
    if sanitize:
        cmd[1:2] = ["-O1", "-g", "-fsanitize=address,undefined", "-fno-omit-frame-pointer"]
    subprocess.run(cmd, check=True)
    return out


def _load():
    global _lib
    if _lib is None:
        # PLE_ORACLE_SANITIZED=1 loads the ASan/UBSan build (the process must
        # then preload the sanitizer runtimes; see tests/test_oracle_pins.py)
        sanitized = os.environ.get("PLE_ORACLE_SANITIZED") == "1"
        path = build(sanitize=sanitized)
        lib = ctypes.CDLL(path)
        lib.oracle_ple_rows.argtypes = [_i64p, ctypes.c_int64, _i32p, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.c_int64, _i64p, _i64p, _i64p, _i64p]
        lib.oracle_ple_rows.restype = ctypes.c_int
        lib.oracle_ple_rows_mt.argtypes = lib.oracle_ple_rows.argtypes + [ctypes.c_int32]
        lib.oracle_ple_rows_mt.restype = ctypes.c_int
        lib.oracle_ple_gather.argtypes = [_i64p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                          ctypes.c_int64, ctypes.c_void_p]
        lib.oracle_ple_gather.restype = ctypes.c_int
        lib.oracle_ple_gather_mt.argtypes = lib.oracle_ple_gather.argtypes + [ctypes.c_int32]
        lib.oracle_ple_gather_mt.restype = ctypes.c_int
        lib.oracle_ple_gather_e4m3.argtypes = [_i64p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                               ctypes.c_int64, ctypes.c_void_p]
        lib.oracle_ple_gather_e4m3.restype = ctypes.c_int
        lib.oracle_ple_count_unique.argtypes = [_i64p, ctypes.c_int64]
        lib.oracle_ple_count_unique.restype = ctypes.c_int64
        lib.oracle_ple_grad_sums.argtypes = [_i64p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int,
                                             ctypes.c_int32, _i64p, _f32p]
        lib.oracle_ple_grad_sums.restype = ctypes.c_int64
        lib.oracle_ple_grad_sums_mt.argtypes = lib.oracle_ple_grad_sums.argtypes + [ctypes.c_int32]
        lib.oracle_ple_grad_sums_mt.restype = ctypes.c_int64
        lib.oracle_ple_grad_apply.argtypes = [_i64p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int,
                                              ctypes.c_int32, ctypes.c_int64, _f32p]
        lib.oracle_ple_grad_apply.restype = ctypes.c_int
        _f64p = ctypes.POINTER(ctypes.c_double)
        lib.oracle_conv_forward.argtypes = [_f64p, ctypes.c_int64, ctypes.c_int64, _i32p, ctypes.c_int32, _f64p,
                                            ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, _f64p]
        lib.oracle_conv_forward.restype = ctypes.c_int
        lib.oracle_conv_backward.argtypes = [_f64p, _f64p, ctypes.c_int64, ctypes.c_int64, _i32p, ctypes.c_int32,
                                             _f64p, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_conv_backward.restype = ctypes.c_int
        _lib = lib
    return _lib


def _p(a, t):
    return a.ctypes.data_as(t)


def rows(tokens, cu_seqlens, ngram_size, heads_per_ngram, eos_id, mults, primes, offsets,
         threads: int = 1) -> np.ndarray:
    """Global table rows ``[T, H]`` (int64) of every (token, head)."""
    tok = np.ascontiguousarray(tokens, dtype=np.int64)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    m = np.ascontiguousarray(mults, dtype=np.int64)
    p = np.ascontiguousarray(primes, dtype=np.int64)
    o = np.ascontiguousarray(offsets, dtype=np.int64)
    H = (ngram_size - 1) * heads_per_ngram
    if m.shape != (ngram_size,) or p.shape != (H,) or o.shape != (H,):
        raise ValueError("mults must be [ngram_size]; primes, offsets [(ngram_size-1)*heads_per_ngram]")
    out = np.empty((tok.shape[0], H), dtype=np.int64)
    args = (_p(tok, _i64p), tok.shape[0], _p(cu, _i32p), cu.shape[0] - 1, ngram_size, heads_per_ngram,
            eos_id, _p(m, _i64p), _p(p, _i64p), _p(o, _i64p), _p(out, _i64p))
    rc = _load().oracle_ple_rows(*args) if threads <= 1 else _load().oracle_ple_rows_mt(*args, threads)
    if rc != 0:
        raise ValueError("malformed cu_seqlens")
    return out


def gather(rows_, table: np.ndarray, threads: int = 1) -> np.ndarray:
    """``out[i] = table[rows[i]]`` as an exact copy; out has shape rows.shape + [D]."""
    r = np.ascontiguousarray(rows_, dtype=np.int64)
    tab = np.ascontiguousarray(table)
    row_bytes = tab.strides[0]
    out = np.empty(r.shape + tab.shape[1:], dtype=tab.dtype)
    args = (_p(r, _i64p), r.size, tab.ctypes.data, tab.shape[0], row_bytes, out.ctypes.data)
    rc = _load().oracle_ple_gather(*args) if threads <= 1 else _load().oracle_ple_gather_mt(*args, threads)
    if rc != 0:
        raise ValueError("row outside the table")
    return out


def gather_e4m3(rows_, table_codes: np.ndarray) -> np.ndarray:
    """Gather from an fp8 e4m3 table (uint8 codes [R, D]) widened to bf16
    (uint16 bit patterns), shape rows.shape + [D]."""
    r = np.ascontiguousarray(rows_, dtype=np.int64)
    tab = np.ascontiguousarray(table_codes, dtype=np.uint8)
    D = tab.shape[1]
    out = np.empty(r.shape + (D,), dtype=np.uint16)
    rc = _load().oracle_ple_gather_e4m3(_p(r, _i64p), r.size, tab.ctypes.data, tab.shape[0], D, out.ctypes.data)
    if rc != 0:
        raise ValueError("row outside the table")
    return out


def lookup(tokens, cu_seqlens, ngram_size, heads_per_ngram, eos_id, mults, primes, offsets, table):
    """Hash then gather: ``[T, H, D]`` values and the ``[T, H]`` rows."""
    r = rows(tokens, cu_seqlens, ngram_size, heads_per_ngram, eos_id, mults, primes, offsets)
    return gather(r, table), r


def slice_positions(num_tokens, row_len, start, end):
    """Packed positions of the slice [start, end) of every row of row_len tokens."""
    if row_len <= 0 or num_tokens % row_len != 0 or not (0 <= start <= end <= row_len):
        raise ValueError("need num_tokens = B * row_len and 0 <= start <= end <= row_len")
    B = num_tokens // row_len
    return (np.arange(B)[:, None] * row_len + np.arange(start, end)[None, :]).reshape(-1)


def lookup_slice(tokens, cu_seqlens, ngram_size, heads_per_ngram, eos_id, mults, primes, offsets, table,
                 row_len, start, end):
    """Global-slice lookup (NeMo engram API page, _forward_global_slice): hash
    the complete packed stream, then gather only the slice [start, end) of
    every row: values [B, end-start, H, D] and rows [B, end-start, H]."""
    r = rows(tokens, cu_seqlens, ngram_size, heads_per_ngram, eos_id, mults, primes, offsets)
    pos = slice_positions(len(tokens), row_len, start, end)
    B = len(tokens) // row_len
    sel = r[pos].reshape(B, end - start, r.shape[1])
    return gather(sel, table), sel


def _grad_args(grad):
    g = np.ascontiguousarray(grad)
    if g.dtype == np.float32:
        return g, 0
    if g.dtype == np.uint16:  # bf16 bit patterns
        return g, 1
    raise ValueError("grad must be float32 or bf16 bits (uint16)")


def grad_sums(rows_, grad, threads: int = 1):
    """Touched rows (ascending) and their fp32 sums in the fixed chunked order."""
    r = np.ascontiguousarray(rows_, dtype=np.int64).reshape(-1)
    g, is_bf16 = _grad_args(grad)
    D = g.shape[-1]
    if g.size != r.size * D:
        raise ValueError("grad must be [N, D] for N rows")
    lib = _load()
    U = lib.oracle_ple_count_unique(_p(r, _i64p), r.size)
    uniq = np.empty(U, dtype=np.int64)
    sums = np.empty((U, D), dtype=np.float32)
    args = (_p(r, _i64p), r.size, g.ctypes.data, is_bf16, D, _p(uniq, _i64p), _p(sums, _f32p))
    got = lib.oracle_ple_grad_sums(*args) if threads <= 1 else lib.oracle_ple_grad_sums_mt(*args, threads)
    assert got == U
    return uniq, sums


def grad_apply(rows_, grad, table_grad: np.ndarray) -> np.ndarray:
    """``table_grad[r] = table_grad[r] + S_r`` in place on a dense fp32 array."""
    r = np.ascontiguousarray(rows_, dtype=np.int64).reshape(-1)
    g, is_bf16 = _grad_args(grad)
    if table_grad.dtype != np.float32 or not table_grad.flags.c_contiguous:
        raise ValueError("table_grad must be a contiguous float32 array")
    D = table_grad.shape[1]
    if g.size != r.size * D:
        raise ValueError("grad must be [N, D] for N rows")
    rc = _load().oracle_ple_grad_apply(_p(r, _i64p), r.size, g.ctypes.data, is_bf16, D,
                                       table_grad.shape[0], _p(table_grad, _f32p))
    if rc != 0:
        raise ValueError("row outside the table")
    return table_grad


# ---------------------------------------------------------------------------
# segment-aware causal dilated depthwise convolution (PLE layer's short conv)
# ---------------------------------------------------------------------------
_f64p = ctypes.POINTER(ctypes.c_double)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def conv_forward(x, cu_seqlens, w, dilation: int, bias=None) -> np.ndarray:
    """y [T, C] of the segment-aware causal dilated depthwise convolution of x [T, C]
    with filters w [C, K] (tap k reads dilation*(K-1-k) tokens back, zero before the
    segment start) plus bias [C]; fp64."""
    x, w = _f64(x), _f64(w)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    T, C = x.shape
    K = w.shape[1]
    b = None if bias is None else _f64(bias)
    y = np.empty((T, C), np.float64)
    rc = _load().oracle_conv_forward(_p(x, _f64p), T, C, _p(cu, _i32p), len(cu) - 1, _p(w, _f64p), K, int(dilation),
                                     None if b is None else b.ctypes.data, _p(y, _f64p))
    if rc != 0:
        raise ValueError(f"bad conv arguments ({rc})")
    return y


def conv_backward(dy, x, cu_seqlens, w, dilation: int):
    """(dx [T, C], dw [C, K], db [C]) of conv_forward for the output gradient dy; fp64."""
    dy, x, w = _f64(dy), _f64(x), _f64(w)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    T, C = x.shape
    K = w.shape[1]
    dx = np.empty((T, C), np.float64)
    dw = np.empty((C, K), np.float64)
    db = np.empty(C, np.float64)
    rc = _load().oracle_conv_backward(_p(dy, _f64p), _p(x, _f64p), T, C, _p(cu, _i32p), len(cu) - 1, _p(w, _f64p),
                                      K, int(dilation), dx.ctypes.data, dw.ctypes.data, db.ctypes.data)
    if rc != 0:
        raise ValueError(f"bad conv arguments ({rc})")
    return dx, dw, db
