"""Thin ctypes binding of libple (include/ple.h).

Argument marshalling only: every step of the lookup runs in the library's
CUDA kernels.  PyTorch supplies device memory (output and workspace tensors
are allocated here with torch when the caller does not pass them) and the
current CUDA stream.  There is no fallback: if libple.so is missing or a
call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

from ._build import LIB_PATH

PLE_OK = 0
PLE_ERR_INVALID_ARG = 1
PLE_ERR_UNSUPPORTED = 2
PLE_ERR_ALIGNMENT = 3
PLE_ERR_WORKSPACE = 4
PLE_ERR_CUDA = 5
PLE_ERR_BAD_ROW = 6
PLE_ERR_BAD_SEQLENS = 7
PLE_ERR_TIMEOUT = 8

PLE_F32 = 0
PLE_BF16 = 1
PLE_F8E4M3 = 2

_DTYPES = {torch.float32: PLE_F32, torch.bfloat16: PLE_BF16}          # tables and gradients
_TABLE_DTYPES = {**_DTYPES, torch.float8_e4m3fn: PLE_F8E4M3}           # tables only
_DTYPE_OF_CODE = {PLE_F32: torch.float32, PLE_BF16: torch.bfloat16, PLE_F8E4M3: torch.float8_e4m3fn}

# every symbol include/ple.h declares
EXPORTS = ("ple_plan_create", "ple_plan_destroy", "ple_plan_num_heads", "ple_hash", "ple_lookup", "ple_lookup_slice",
           "ple_gather",
           "ple_grad_scatter_workspace_bytes", "ple_grad_scatter", "ple_grad_prepare", "ple_grad_apply",
           "ple_grad_scatter_atomic",
           "ple_grad_scatter_noalloc", "ple_grad_scatter_noalloc_scratch_bytes", "ple_prefetch_workspace_bytes",
           "ple_prefetch", "ple_gather_cache", "ple_grad_scatter_cache", "ple_conv_forward",
           "ple_conv_backward_workspace_bytes", "ple_conv_backward", "ple_status", "ple_strerror",
           "ple_last_cuda_error",
           # include/ple_debug.h
           "ple_debug_set_wait_limit_ns", "ple_debug_default_wait_limit_ns")


class PleError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib().ple_strerror(status).decode()
        if status == PLE_ERR_CUDA:
            msg += f" (cudaError {_lib().ple_last_cuda_error()})"
        super().__init__(f"{where}: {msg} [status {status}]")


class _Params(ctypes.Structure):
    _fields_ = [("ngram_size", ctypes.c_int32), ("heads_per_ngram", ctypes.c_int32), ("eos_id", ctypes.c_int64),
                ("mults", ctypes.POINTER(ctypes.c_int64)), ("primes", ctypes.POINTER(ctypes.c_int64)),
                ("offsets", ctypes.POINTER(ctypes.c_int64)), ("num_rows", ctypes.c_int64),
                ("head_dim", ctypes.c_int32), ("table_dtype", ctypes.c_int)]


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libple is not built ({LIB_PATH}); run __graft_entry__.build() or "
                              "python -m hashed_gram_embedding_ple_b200._build")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        lib.ple_plan_create.argtypes = [ctypes.POINTER(_Params), ctypes.POINTER(vp)]
        lib.ple_plan_destroy.argtypes = [vp]
        lib.ple_plan_destroy.restype = None
        lib.ple_plan_num_heads.argtypes = [vp]
        lib.ple_plan_num_heads.restype = i32
        lib.ple_hash.argtypes = [vp, vp, i64, vp, i32, vp, vp]
        lib.ple_lookup.argtypes = [vp, vp, i64, vp, i32, vp, vp, vp, vp]
        lib.ple_lookup_slice.argtypes = [vp, vp, i64, vp, i32, i64, i64, i64, vp, vp, vp, vp]
        lib.ple_gather.argtypes = [vp, vp, i64, vp, vp, vp]
        lib.ple_grad_scatter_workspace_bytes.argtypes = [vp, i64]
        lib.ple_grad_scatter_workspace_bytes.restype = sz
        lib.ple_grad_scatter.argtypes = [vp, vp, i64, vp, ctypes.c_int, vp, vp, sz, vp]
        lib.ple_grad_prepare.argtypes = [vp, vp, i64, vp, sz, vp]
        lib.ple_grad_apply.argtypes = [vp, i64, vp, ctypes.c_int, vp, vp, sz, vp]
        lib.ple_grad_scatter_atomic.argtypes = [vp, vp, i64, vp, ctypes.c_int, vp, vp]
        lib.ple_grad_scatter_noalloc.argtypes = [vp, vp, i64, vp, ctypes.c_int, vp, vp]
        lib.ple_grad_scatter_noalloc_scratch_bytes.argtypes = []
        lib.ple_grad_scatter_noalloc_scratch_bytes.restype = sz
        lib.ple_prefetch_workspace_bytes.argtypes = [vp, i64]
        lib.ple_prefetch_workspace_bytes.restype = sz
        lib.ple_prefetch.argtypes = [vp, vp, i64, vp, i32, vp, vp, i64, vp, vp, vp, vp, sz, vp]
        lib.ple_gather_cache.argtypes = [vp, vp, i64, vp, i64, vp, vp]
        lib.ple_grad_scatter_cache.argtypes = [vp, vp, i64, vp, ctypes.c_int, vp, i64, vp, sz, vp]
        lib.ple_conv_forward.argtypes = [vp, ctypes.c_int, i64, i64, vp, i32, vp, i32, i32, vp, vp, vp]
        lib.ple_conv_backward_workspace_bytes.argtypes = [i64, i64, i32]
        lib.ple_conv_backward_workspace_bytes.restype = sz
        lib.ple_conv_backward.argtypes = [vp, vp, ctypes.c_int, i64, i64, vp, i32, vp, i32, i32, vp, vp, vp, vp, sz,
                                          vp]
        lib.ple_status.argtypes = [vp, vp]
        lib.ple_strerror.argtypes = [ctypes.c_int]
        lib.ple_strerror.restype = ctypes.c_char_p
        lib.ple_last_cuda_error.argtypes = []
        lib.ple_debug_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        lib.ple_debug_set_wait_limit_ns.restype = ctypes.c_uint64
        lib.ple_debug_default_wait_limit_ns.argtypes = []
        lib.ple_debug_default_wait_limit_ns.restype = ctypes.c_uint64
        for name in ("ple_plan_create", "ple_hash", "ple_lookup", "ple_lookup_slice", "ple_gather", "ple_grad_scatter",
                     "ple_grad_prepare", "ple_grad_apply",
                     "ple_grad_scatter_atomic", "ple_grad_scatter_noalloc", "ple_prefetch", "ple_gather_cache",
                     "ple_grad_scatter_cache", "ple_conv_forward",
                     "ple_conv_backward", "ple_status", "ple_last_cuda_error"):
            getattr(lib, name).restype = ctypes.c_int
        _LIB = lib
    return _LIB


def lib():
    """The loaded libple CDLL (raises ImportError if it is not built)."""
    return _lib()


def _check(rc: int, where: str):
    if rc != PLE_OK:
        raise PleError(rc, where)


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


class Plan:
    """Hash and table description (ple_params_t) validated by ple_plan_create."""

    def __init__(self, ngram_size, heads_per_ngram, eos_id, mults, primes, offsets, num_rows, head_dim,
                 table_dtype=torch.bfloat16):
        H = (ngram_size - 1) * heads_per_ngram
        self._mults = (ctypes.c_int64 * max(1, len(mults)))(*[int(m) for m in mults])
        self._primes = (ctypes.c_int64 * max(1, len(primes)))(*[int(p) for p in primes])
        self._offsets = (ctypes.c_int64 * max(1, len(offsets)))(*[int(o) for o in offsets])
        if len(mults) != ngram_size or len(primes) != H or len(offsets) != H:
            raise ValueError("mults must have ngram_size entries; primes and offsets (ngram_size-1)*heads_per_ngram")
        if table_dtype not in _TABLE_DTYPES:
            raise ValueError(f"table dtype must be float32, bfloat16 or float8_e4m3fn, not {table_dtype}")
        p = _Params(ngram_size, heads_per_ngram, int(eos_id), self._mults, self._primes, self._offsets,
                    int(num_rows), int(head_dim), _TABLE_DTYPES[table_dtype])
        handle = ctypes.c_void_p()
        _check(_lib().ple_plan_create(ctypes.byref(p), ctypes.byref(handle)), "ple_plan_create")
        self._h = handle
        self.ngram_size, self.heads_per_ngram, self.num_heads = ngram_size, heads_per_ngram, H
        self.num_rows, self.head_dim, self.table_dtype = int(num_rows), int(head_dim), table_dtype
        # lookups of an fp8 table are widened to bf16
        self.out_dtype = torch.bfloat16 if table_dtype == torch.float8_e4m3fn else table_dtype

    @classmethod
    def from_workload(cls, w):
        return cls(w.ngram_size, w.heads_per_ngram, w.eos_id, w.mults, w.primes, w.offsets, w.num_rows,
                   w.head_dim, _DTYPE_OF_CODE[w.table_dtype])

    @property
    def handle(self):
        return self._h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _LIB is not None:
            _LIB.ple_plan_destroy(h)
            self._h = None


def _as_i64(t, name):
    if t.dtype != torch.int64 or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name} must be a contiguous int64 CUDA tensor")


def _as_i32(t, name):
    if t.dtype != torch.int32 or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name} must be a contiguous int32 CUDA tensor")


def _check_table(plan: Plan, table):
    if table.dtype != plan.table_dtype or not table.is_contiguous() or table.shape[-1] != plan.head_dim \
            or table.numel() != plan.num_rows * plan.head_dim or not table.is_cuda:
        raise ValueError("table must be a contiguous CUDA tensor [num_rows, head_dim] in the plan's dtype")


def _out(plan: Plan, out, shape, device):
    """The caller's output tensor, checked, or a new one."""
    if out is None:
        return torch.empty(*shape, dtype=plan.out_dtype, device=device)
    n = 1
    for d in shape:
        n *= d
    if out.dtype != plan.out_dtype or not out.is_contiguous() or out.numel() != n or out.device != device:
        raise ValueError(f"out must be a contiguous {plan.out_dtype} tensor of {n} elements on {device}")
    return out


def _rows(rows, shape, device):
    n = 1
    for d in shape:
        n *= d
    if rows.dtype != torch.int64 or not rows.is_contiguous() or rows.numel() != n or rows.device != device:
        raise ValueError(f"rows_out must be a contiguous int64 tensor of {n} elements on {device}")
    return rows


def ple_hash(plan: Plan, tokens, cu_seqlens, rows=None):
    """int64 [T, H] global rows of every (token, head)."""
    _as_i64(tokens, "tokens")
    _as_i32(cu_seqlens, "cu_seqlens")
    T = tokens.numel()
    if rows is None:
        rows = torch.empty(T, plan.num_heads, dtype=torch.int64, device=tokens.device)
    else:
        _rows(rows, (T, plan.num_heads), tokens.device)
    _check(_lib().ple_hash(plan.handle, _ptr(tokens), T, _ptr(cu_seqlens), cu_seqlens.numel() - 1, _ptr(rows),
                           _stream(tokens.device)), "ple_hash")
    return rows


def ple_lookup(plan: Plan, tokens, cu_seqlens, table, out=None, rows_out=None, save_rows: bool = False):
    """Hash fused with the gather: [T, H, D] values in the table dtype (bf16
    for an fp8 table).  With save_rows (or a rows_out tensor) also returns the
    [T, H] rows."""
    _as_i64(tokens, "tokens")
    _as_i32(cu_seqlens, "cu_seqlens")
    _check_table(plan, table)
    T = tokens.numel()
    out = _out(plan, out, (T, plan.num_heads, plan.head_dim), table.device)
    if rows_out is None and save_rows:
        rows_out = torch.empty(T, plan.num_heads, dtype=torch.int64, device=tokens.device)
    elif rows_out is not None:
        _rows(rows_out, (T, plan.num_heads), tokens.device)
    _check(_lib().ple_lookup(plan.handle, _ptr(tokens), T, _ptr(cu_seqlens), cu_seqlens.numel() - 1,
                             _ptr(table), _ptr(out), _ptr(rows_out), _stream(tokens.device)), "ple_lookup")
    return (out, rows_out) if rows_out is not None else out


def ple_lookup_slice(plan: Plan, tokens, cu_seqlens, row_len: int, start: int, end: int, table, out=None,
                     rows_out=None, save_rows: bool = False):
    """Global-slice lookup: [B, end-start, H, D] values of positions
    [start, end) of every row of row_len tokens, hashed with full context."""
    _as_i64(tokens, "tokens")
    _as_i32(cu_seqlens, "cu_seqlens")
    _check_table(plan, table)
    T = tokens.numel()
    if row_len < 1 or T % row_len != 0 or not (0 <= start <= end <= row_len):
        raise ValueError("need num_tokens = B * row_len and 0 <= start <= end <= row_len")
    B, W = T // row_len, end - start
    out = _out(plan, out, (B, W, plan.num_heads, plan.head_dim), table.device)
    if rows_out is None and save_rows:
        rows_out = torch.empty(B, W, plan.num_heads, dtype=torch.int64, device=tokens.device)
    elif rows_out is not None:
        _rows(rows_out, (B, W, plan.num_heads), tokens.device)
    _check(_lib().ple_lookup_slice(plan.handle, _ptr(tokens), T, _ptr(cu_seqlens), cu_seqlens.numel() - 1, row_len,
                                   start, end, _ptr(table), _ptr(out), _ptr(rows_out), _stream(tokens.device)),
           "ple_lookup_slice")
    return (out, rows_out) if rows_out is not None else out


def ple_gather(plan: Plan, rows, table, out=None):
    """out[i] = table[rows[i]] for flat rows; shape rows.shape + [D] (bf16
    for an fp8 table)."""
    _as_i64(rows, "rows")
    _check_table(plan, table)
    out = _out(plan, out, (*rows.shape, plan.head_dim), table.device)
    _check(_lib().ple_gather(plan.handle, _ptr(rows), rows.numel(), _ptr(table), _ptr(out),
                             _stream(rows.device)), "ple_gather")
    return out


def workspace_bytes(plan: Plan, num_hits: int) -> int:
    return int(_lib().ple_grad_scatter_workspace_bytes(plan.handle, int(num_hits)))


def alloc_workspace(plan: Plan, num_hits: int, device):
    n = workspace_bytes(plan, num_hits)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device)


def _grad_dtype(g):
    if g.dtype not in _DTYPES or not g.is_contiguous():
        raise ValueError("grad_out must be contiguous float32 or bfloat16")
    return _DTYPES[g.dtype]


def _check_table_grad(plan: Plan, table_grad):
    if table_grad.dtype != torch.float32 or not table_grad.is_contiguous() or not table_grad.is_cuda \
            or table_grad.numel() != plan.num_rows * plan.head_dim:
        raise ValueError("table_grad must be a contiguous float32 CUDA tensor [num_rows, head_dim]")


def ple_grad_scatter(plan: Plan, rows, grad_out, table_grad, workspace=None):
    """Deterministic table_grad += per-row sums of grad_out (fixed chunked order)."""
    _as_i64(rows, "rows")
    gdt = _grad_dtype(grad_out)
    _check_table_grad(plan, table_grad)
    N = rows.numel()
    if grad_out.numel() != N * plan.head_dim:
        raise ValueError("grad_out must hold num_hits * head_dim values")
    if workspace is None:
        workspace = alloc_workspace(plan, N, rows.device)
    _check(_lib().ple_grad_scatter(plan.handle, _ptr(rows), N, _ptr(grad_out), gdt, _ptr(table_grad),
                                   _ptr(workspace), workspace.numel(), _stream(rows.device)), "ple_grad_scatter")
    return table_grad


def ple_grad_prepare(plan: Plan, rows, workspace):
    """First half of ple_grad_scatter: sort the rows into the workspace (it
    must then stay untouched until the matching ple_grad_apply)."""
    _as_i64(rows, "rows")
    N = rows.numel()
    _check(_lib().ple_grad_prepare(plan.handle, _ptr(rows), N, _ptr(workspace), workspace.numel(),
                                   _stream(rows.device)), "ple_grad_prepare")
    return workspace


def ple_grad_apply(plan: Plan, num_hits: int, grad_out, table_grad, workspace):
    """Second half: fold grad_out in the prepared order into table_grad."""
    gdt = _grad_dtype(grad_out)
    _check_table_grad(plan, table_grad)
    if grad_out.numel() != int(num_hits) * plan.head_dim:
        raise ValueError("grad_out must hold num_hits * head_dim values")
    _check(_lib().ple_grad_apply(plan.handle, int(num_hits), _ptr(grad_out), gdt, _ptr(table_grad), _ptr(workspace),
                                 workspace.numel(), _stream(grad_out.device)), "ple_grad_apply")
    return table_grad


def ple_grad_scatter_atomic(plan: Plan, rows, grad_out, table_grad):
    """Non-deterministic fp32 atomic variant (speed reference)."""
    _as_i64(rows, "rows")
    gdt = _grad_dtype(grad_out)
    _check_table_grad(plan, table_grad)
    N = rows.numel()
    if grad_out.numel() != N * plan.head_dim:
        raise ValueError("grad_out must hold num_hits * head_dim values")
    _check(_lib().ple_grad_scatter_atomic(plan.handle, _ptr(rows), N, _ptr(grad_out), gdt, _ptr(table_grad),
                                          _stream(rows.device)), "ple_grad_scatter_atomic")
    return table_grad


def ple_grad_scatter_noalloc(plan: Plan, rows, grad_out, table_grad):
    """Deterministic gradient using the library's fixed scratch area (no
    workspace, no allocation); see include/ple.h for the size limit and the
    rules on overlapping calls."""
    _as_i64(rows, "rows")
    gdt = _grad_dtype(grad_out)
    _check_table_grad(plan, table_grad)
    N = rows.numel()
    if grad_out.numel() != N * plan.head_dim:
        raise ValueError("grad_out must hold num_hits * head_dim values")
    _check(_lib().ple_grad_scatter_noalloc(plan.handle, _ptr(rows), N, _ptr(grad_out), gdt, _ptr(table_grad),
                                           _stream(rows.device)), "ple_grad_scatter_noalloc")
    return table_grad


# ---------------------------------------------------------------------------
# host-memory tier: table in pinned host memory, distinct rows prefetched
# ---------------------------------------------------------------------------

class Prefetched:
    """Device buffers of one prefetched batch: cache [cache_rows, D], slots
    [T, H], uniq_rows [cache_rows], num_unique (one int64 on the device)."""

    def __init__(self, plan: Plan, num_tokens: int, device):
        n = int(num_tokens) * plan.num_heads
        self.cache_rows = max(n, 1)
        self.cache = torch.empty(self.cache_rows, plan.head_dim, dtype=plan.table_dtype, device=device)
        self.slots = torch.empty(int(num_tokens), plan.num_heads, dtype=torch.int64, device=device)
        self.uniq_rows = torch.empty(self.cache_rows, dtype=torch.int64, device=device)
        self.num_unique = torch.zeros(1, dtype=torch.int64, device=device)
        self.workspace = torch.empty(max(int(_lib().ple_prefetch_workspace_bytes(plan.handle, int(num_tokens))), 1),
                                     dtype=torch.uint8, device=device)


def ple_prefetch(plan: Plan, tokens, cu_seqlens, host_table, buffers: "Prefetched" = None):
    """Hash the batch and copy each distinct row once from host_table (a
    pinned CPU tensor [num_rows, D] in the plan's dtype) into a device cache.
    Runs on the current stream; returns the Prefetched buffers."""
    _as_i64(tokens, "tokens")
    _as_i32(cu_seqlens, "cu_seqlens")
    if host_table.dtype != plan.table_dtype or not host_table.is_contiguous() or host_table.is_cuda \
            or not host_table.is_pinned() or host_table.numel() != plan.num_rows * plan.head_dim:
        raise ValueError("host_table must be a contiguous pinned CPU tensor [num_rows, head_dim] in the plan's dtype")
    T = tokens.numel()
    if buffers is None:
        buffers = Prefetched(plan, T, tokens.device)
    elif buffers.slots.numel() != T * plan.num_heads:
        raise ValueError("buffers were made for another number of tokens")
    _check(_lib().ple_prefetch(plan.handle, _ptr(tokens), T, _ptr(cu_seqlens), cu_seqlens.numel() - 1,
                               host_table.data_ptr(), _ptr(buffers.cache), buffers.cache_rows, _ptr(buffers.slots),
                               _ptr(buffers.uniq_rows), _ptr(buffers.num_unique), _ptr(buffers.workspace),
                               buffers.workspace.numel(), _stream(tokens.device)), "ple_prefetch")
    return buffers


def ple_gather_cache(plan: Plan, buffers: "Prefetched", out=None):
    """The lookup of a prefetched batch: [T, H, D] (bf16 for an fp8 table)."""
    T, H = buffers.slots.shape
    out = _out(plan, out, (T, H, plan.head_dim), buffers.cache.device)
    _check(_lib().ple_gather_cache(plan.handle, _ptr(buffers.slots), T * H, _ptr(buffers.cache), buffers.cache_rows,
                                   _ptr(out), _stream(out.device)), "ple_gather_cache")
    return out


def ple_grad_scatter_cache(plan: Plan, buffers: "Prefetched", grad_out, cache_grad=None, workspace=None):
    """Deterministic gradient of a prefetched batch into cache_grad fp32
    [cache_rows, D] (accumulated into; row u belongs to uniq_rows[u])."""
    gdt = _grad_dtype(grad_out)
    N = buffers.slots.numel()
    if grad_out.numel() != N * plan.head_dim:
        raise ValueError("grad_out must hold num_hits * head_dim values")
    dev = buffers.cache.device
    if cache_grad is None:
        cache_grad = torch.zeros(buffers.cache_rows, plan.head_dim, dtype=torch.float32, device=dev)
    elif cache_grad.dtype != torch.float32 or cache_grad.numel() != buffers.cache_rows * plan.head_dim \
            or not cache_grad.is_contiguous():
        raise ValueError("cache_grad must be a contiguous float32 tensor [cache_rows, head_dim]")
    if workspace is None:
        workspace = alloc_workspace(plan, N, dev)
    _check(_lib().ple_grad_scatter_cache(plan.handle, _ptr(buffers.slots), N, _ptr(grad_out), gdt, _ptr(cache_grad),
                                         buffers.cache_rows, _ptr(workspace), workspace.numel(), _stream(dev)),
           "ple_grad_scatter_cache")
    return cache_grad


# ---------------------------------------------------------------------------
# the PLE layer's short convolution (segment-aware, causal, dilated, depthwise)
# ---------------------------------------------------------------------------

def _conv_check(x, cu_seqlens, weight):
    if x.dim() != 2 or x.dtype not in _DTYPES or not x.is_contiguous() or not x.is_cuda:
        raise ValueError("x must be a contiguous [tokens, channels] float32 or bfloat16 CUDA tensor")
    _as_i32(cu_seqlens, "cu_seqlens")
    if weight.dtype != torch.float32 or not weight.is_contiguous() or weight.dim() != 2 \
            or weight.shape[0] != x.shape[1] or not weight.is_cuda:
        raise ValueError("weight must be a contiguous float32 CUDA tensor [channels, kernel_size]")


def conv_forward(x, cu_seqlens, weight, dilation: int, bias=None, out=None):
    """y = segment-aware causal dilated depthwise convolution of x [T, C] with
    weight [C, K] (+ bias [C]); y has x's shape and dtype."""
    _conv_check(x, cu_seqlens, weight)
    T, C = x.shape
    if bias is not None and (bias.dtype != torch.float32 or bias.numel() != C or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous float32 tensor [channels]")
    if out is None:
        out = torch.empty_like(x)
    elif out.shape != x.shape or out.dtype != x.dtype or not out.is_contiguous():
        raise ValueError("out must match x")
    _check(_lib().ple_conv_forward(_ptr(x), _DTYPES[x.dtype], T, C, _ptr(cu_seqlens), cu_seqlens.numel() - 1,
                                   _ptr(weight), weight.shape[1], int(dilation), _ptr(bias), _ptr(out),
                                   _stream(x.device)), "ple_conv_forward")
    return out


def conv_workspace_bytes(num_tokens: int, channels: int, kernel_size: int) -> int:
    return int(_lib().ple_conv_backward_workspace_bytes(int(num_tokens), int(channels), int(kernel_size)))


def conv_backward(dy, x, cu_seqlens, weight, dilation: int, dx=None, want_dx: bool = True, dweight=None,
                  dbias=None, workspace=None):
    """Gradients of conv_forward: returns (dx, dweight, dbias).  dx is
    written (allocated unless given; skipped with want_dx=False); dweight
    [C, K] and dbias [C] are fp32 tensors accumulated into when given."""
    _conv_check(x, cu_seqlens, weight)
    if dy.shape != x.shape or dy.dtype != x.dtype or not dy.is_contiguous():
        raise ValueError("dy must match x")
    T, C = x.shape
    K = weight.shape[1]
    if dx is None and want_dx:
        dx = torch.empty_like(x)
    elif dx is not None and (dx.shape != x.shape or dx.dtype != x.dtype or not dx.is_contiguous()):
        raise ValueError("dx must match x")
    for name, t, n in (("dweight", dweight, C * K), ("dbias", dbias, C)):
        if t is not None and (t.dtype != torch.float32 or t.numel() != n or not t.is_contiguous() or not t.is_cuda):
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor of {n} elements")
    if (dweight is not None or dbias is not None) and workspace is None:
        workspace = torch.empty(max(conv_workspace_bytes(T, C, K), 1), dtype=torch.uint8, device=x.device)
    _check(_lib().ple_conv_backward(_ptr(dy), _ptr(x), _DTYPES[x.dtype], T, C, _ptr(cu_seqlens),
                                    cu_seqlens.numel() - 1, _ptr(weight), K, int(dilation), _ptr(dx), _ptr(dweight),
                                    _ptr(dbias), _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                    _stream(x.device)), "ple_conv_backward")
    return dx, dweight, dbias


def set_wait_limit_ns(ns: int) -> int:
    """Limit of the bounded waits between blocks for later calls (every
    device, this process); returns the previous limit (include/ple_debug.h)."""
    return int(_lib().ple_debug_set_wait_limit_ns(int(ns)))


def default_wait_limit_ns() -> int:
    return int(_lib().ple_debug_default_wait_limit_ns())


def noalloc_scratch_bytes() -> int:
    return int(_lib().ple_grad_scatter_noalloc_scratch_bytes())


def ple_status(device=None, plan: Plan = None) -> int:
    """Take (return and clear) the async status on the current stream: the
    word of `plan`, or with no plan every word of the device (all plans and
    the plan-less calls)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    return int(_lib().ple_status(None if plan is None else plan.handle, _stream(dev)))
