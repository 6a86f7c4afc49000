"""libple's C ABI on the host: the library loads, exports every symbol that
include/ple.h declares, and rejects bad arguments before touching a GPU
(every call below returns on a host check, so no device is needed)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

import hashed_gram_embedding_ple_b200 as ple
from hashed_gram_embedding_ple_b200 import binding


def _declared():
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(ple_[a-z_]+)\s*\(", text))
    return sorted(names)


def test_header_symbols_exported():
    lib = ple.lib()
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(binding.EXPORTS) == names


def test_library_is_in_tree_and_built_for_sm100a():
    path = binding.LIB_PATH
    assert os.path.dirname(path).endswith("hashed_gram_embedding_ple_b200")
    assert os.path.exists(path)


def _plan(**kw):
    args = dict(ngram_size=3, heads_per_ngram=2, eos_id=0, mults=[1, 2, 3], primes=[7, 11, 13, 17],
                offsets=[0, 7, 18, 31], num_rows=48, head_dim=8, table_dtype=binding.torch.bfloat16)
    args.update(kw)
    return ple.Plan(**args)


def test_plan_accepts_valid():
    p = _plan()
    assert ple.lib().ple_plan_num_heads(p.handle) == 4
    q = _plan(head_dim=16, table_dtype=binding.torch.float8_e4m3fn)  # 16 codes = one 16-byte vector
    assert q.out_dtype == binding.torch.bfloat16
    with pytest.raises(ValueError):
        _plan(table_dtype=binding.torch.float16)


@pytest.mark.parametrize("kw,code", [
    (dict(ngram_size=1, mults=[1], primes=[], offsets=[]), binding.PLE_ERR_INVALID_ARG),
    (dict(ngram_size=9, heads_per_ngram=1, mults=[1] * 9, primes=list(range(101, 109)),
          offsets=[0] * 8), binding.PLE_ERR_INVALID_ARG),
    (dict(primes=[7, 1, 13, 17]), binding.PLE_ERR_INVALID_ARG),
    (dict(offsets=[0, 6, 18, 31]), binding.PLE_ERR_INVALID_ARG),          # overlapping ranges
    (dict(offsets=[0, 7, 18, 32]), binding.PLE_ERR_INVALID_ARG),          # past num_rows
    (dict(offsets=[-1, 7, 18, 31]), binding.PLE_ERR_INVALID_ARG),
    (dict(primes=[7, 11, 13, 2 ** 62 + 1], num_rows=2 ** 63 - 1), binding.PLE_ERR_INVALID_ARG),
    (dict(head_dim=4), binding.PLE_ERR_ALIGNMENT),                          # 8-byte rows
    (dict(head_dim=8, table_dtype=binding.torch.float8_e4m3fn), binding.PLE_ERR_ALIGNMENT),  # 8 fp8 codes
    (dict(head_dim=0), binding.PLE_ERR_INVALID_ARG),
    (dict(heads_per_ngram=33, mults=[1, 2, 3], primes=[5] * 66, offsets=[0] * 66), binding.PLE_ERR_UNSUPPORTED),
])
def test_plan_rejects(kw, code):
    with pytest.raises(ple.PleError) as ei:
        _plan(**kw)
    assert ei.value.status == code


def test_plan_rejects_null_params():
    lib = ple.lib()
    out = ctypes.c_void_p()
    assert lib.ple_plan_create(None, ctypes.byref(out)) == binding.PLE_ERR_INVALID_ARG
    assert out.value is None


def test_calls_reject_bad_arguments_on_host():
    lib = ple.lib()
    p = _plan()
    h = p.handle
    # empty input is a no-op
    assert lib.ple_hash(h, None, 0, None, 0, None, None) == 0
    assert lib.ple_lookup(h, None, 0, None, 0, None, None, None, None) == 0
    assert lib.ple_gather(h, None, 0, None, None, None) == 0
    assert lib.ple_grad_scatter(h, None, 0, None, 1, None, None, 0, None) == 0
    # null / negative / misaligned
    assert lib.ple_hash(h, None, 5, 0x1000, 1, 0x2000, None) == binding.PLE_ERR_INVALID_ARG
    assert lib.ple_hash(h, 0x1000, -1, 0x1000, 1, 0x2000, None) == binding.PLE_ERR_INVALID_ARG
    assert lib.ple_hash(h, 0x1000, 5, 0x1000, 0, 0x2000, None) == binding.PLE_ERR_INVALID_ARG
    assert lib.ple_hash(h, 0x1004, 5, 0x1000, 1, 0x2000, None) == binding.PLE_ERR_ALIGNMENT
    assert lib.ple_lookup(h, 0x1000, 5, 0x1000, 1, 0x3008, 0x4000, None, None) == binding.PLE_ERR_ALIGNMENT
    assert lib.ple_lookup(h, 0x1000, 5, 0x1000, 1, 0x3000, 0x4000, 0x5004, None) == binding.PLE_ERR_ALIGNMENT
    assert lib.ple_gather(h, 0x1000, 5, 0x3000, 0x4008, None) == binding.PLE_ERR_ALIGNMENT
    assert lib.ple_gather(h, None, 5, 0x3000, 0x4000, None) == binding.PLE_ERR_INVALID_ARG
    # grad: bad dtype, workspace too small, misaligned workspace
    assert lib.ple_grad_scatter(h, 0x1000, 5, 0x2000, 7, 0x3000, 0x4000, 1 << 20, None) == \
        binding.PLE_ERR_INVALID_ARG
    need = lib.ple_grad_scatter_workspace_bytes(h, 5)
    assert need > 0
    assert lib.ple_grad_scatter(h, 0x1000, 5, 0x2000, 1, 0x3000, 0x4000, need - 1, None) == binding.PLE_ERR_WORKSPACE
    assert lib.ple_grad_scatter(h, 0x1000, 5, 0x2000, 1, 0x3000, None, need, None) == binding.PLE_ERR_WORKSPACE
    assert lib.ple_grad_scatter(h, 0x1000, 5, 0x2000, 1, 0x3000, 0x4010, need, None) == binding.PLE_ERR_ALIGNMENT
    assert lib.ple_grad_scatter(h, 0x1000, 5, 0x2008, 1, 0x3000, 0x4000, need, None) == binding.PLE_ERR_ALIGNMENT
    assert lib.ple_grad_scatter(h, 0x1000, 2 ** 31, 0x2000, 1, 0x3000, 0x4000, 1 << 62, None) == \
        binding.PLE_ERR_UNSUPPORTED
    assert lib.ple_grad_scatter_atomic(h, None, 5, 0x2000, 1, 0x3000, None) == binding.PLE_ERR_INVALID_ARG
    # global slice: row_len must divide num_tokens, 0 <= start <= end <= row_len; empty slice is a no-op
    sl = lib.ple_lookup_slice
    assert sl(h, 0x1000, 12, 0x1000, 1, 5, 0, 2, 0x3000, 0x4000, None, None) == binding.PLE_ERR_INVALID_ARG
    assert sl(h, 0x1000, 12, 0x1000, 1, 4, 3, 2, 0x3000, 0x4000, None, None) == binding.PLE_ERR_INVALID_ARG
    assert sl(h, 0x1000, 12, 0x1000, 1, 4, 0, 5, 0x3000, 0x4000, None, None) == binding.PLE_ERR_INVALID_ARG
    assert sl(h, 0x1000, 12, 0x1000, 1, 4, 2, 2, 0x3000, 0x4000, None, None) == 0
    assert sl(h, 0x1000, 12, 0x1000, 1, 4, 0, 2, 0x3008, 0x4000, None, None) == binding.PLE_ERR_ALIGNMENT


def test_workspace_grows_with_hits():
    p = _plan(head_dim=128)
    a = ple.workspace_bytes(p, 1000)
    b = ple.workspace_bytes(p, 100000)
    assert 0 < a < b
    assert ple.workspace_bytes(p, 0) == 0
    # keys/values double buffers plus chunk-sum slots dominate: roughly 16 B + 2*D*4/32 B per hit
    assert b >= 100000 * (16 + 2 * 128 * 4 // 32)


def test_workspace_never_shrinks_as_hits_grow():
    """A workspace sized for N hits serves every smaller N, across the sort's
    switch from 2048-key to 4096-key tiles (at 3 * 2^17 keys) too."""
    for D in (16, 64, 128):
        p = _plan(head_dim=D)
        ns = sorted({1, 31, 32, 33, 2047, 2048, 2049, 65535, 65536, 3 * 2**17 - 4097, 3 * 2**17 - 1, 3 * 2**17,
                     3 * 2**17 + 1, 3 * 2**17 + 4096, 524288, 1 << 21, (1 << 21) + 1})
        sizes = [ple.workspace_bytes(p, n) for n in ns]
        assert all(a <= b for a, b in zip(sizes, sizes[1:])), list(zip(ns, sizes))
        host = [ple.lib().ple_prefetch_workspace_bytes(p.handle, n) for n in ns]
        assert all(a <= b for a, b in zip(host, host[1:]))


def test_strerror_covers_codes():
    lib = ple.lib()
    for c in range(9):
        assert lib.ple_strerror(c)
    assert b"unknown" in lib.ple_strerror(99)


def test_conv_rejects_bad_arguments_on_host():
    lib = ple.lib()
    f, b = lib.ple_conv_forward, lib.ple_conv_backward
    BF = binding.PLE_BF16
    # empty input is a no-op
    assert f(None, BF, 0, 8, None, 0, None, 4, 3, None, None, None) == 0
    # bad sizes / kinds
    assert f(0x1000, BF, 5, 8, 0x2000, 1, 0x3000, 0, 3, None, 0x4000, None) == binding.PLE_ERR_INVALID_ARG
    assert f(0x1000, BF, 5, 8, 0x2000, 1, 0x3000, 4, 0, None, 0x4000, None) == binding.PLE_ERR_INVALID_ARG
    assert f(0x1000, 7, 5, 8, 0x2000, 1, 0x3000, 4, 3, None, 0x4000, None) == binding.PLE_ERR_INVALID_ARG
    assert f(0x1000, BF, 5, 8, 0x2000, 1, 0x3000, 9, 3, None, 0x4000, None) == binding.PLE_ERR_UNSUPPORTED
    assert f(0x1000, BF, 5, 8, None, 1, 0x3000, 4, 3, None, 0x4000, None) == binding.PLE_ERR_INVALID_ARG
    assert f(0x1000, BF, 5, 8, 0x2000, 1, 0x3000, 4, 3, None, None, None) == binding.PLE_ERR_INVALID_ARG
    # alignment: 8-byte rows, misaligned x / y
    assert f(0x1000, BF, 5, 4, 0x2000, 1, 0x3000, 4, 3, None, 0x4000, None) == binding.PLE_ERR_ALIGNMENT
    assert f(0x1008, BF, 5, 8, 0x2000, 1, 0x3000, 4, 3, None, 0x4000, None) == binding.PLE_ERR_ALIGNMENT
    assert f(0x1000, BF, 5, 8, 0x2000, 1, 0x3000, 4, 3, None, 0x4008, None) == binding.PLE_ERR_ALIGNMENT
    # backward: parameter gradients need the workspace
    need = lib.ple_conv_backward_workspace_bytes(5, 8, 4)
    assert need >= 5 * 8 * 4 * 0 + 8 * 5 * 4
    assert b(0x5000, 0x1000, BF, 5, 8, 0x2000, 1, 0x3000, 4, 3, None, 0x6000, None, None, 0, None) == \
        binding.PLE_ERR_WORKSPACE
    assert b(0x5000, 0x1000, BF, 5, 8, 0x2000, 1, 0x3000, 4, 3, None, 0x6000, None, 0x7000, need - 1, None) == \
        binding.PLE_ERR_WORKSPACE
    assert b(0x5000, 0x1000, BF, 5, 8, 0x2000, 1, 0x3000, 4, 3, None, None, None, None, 0, None) == 0  # nothing asked
    assert b(0x5008, 0x1000, BF, 5, 8, 0x2000, 1, 0x3000, 4, 3, 0x8000, None, None, None, 0, None) == \
        binding.PLE_ERR_ALIGNMENT
    # 1024 chunks at most: the workspace stops growing with the token count past 256 K tokens
    assert lib.ple_conv_backward_workspace_bytes(1 << 24, 8, 4) == 1024 * 8 * 5 * 4


def test_host_tier_rejects_bad_arguments_on_host():
    lib = ple.lib()
    p = _plan()  # 4 heads
    h = p.handle
    pf = lib.ple_prefetch
    # empty: only the device count is written -> needs a count pointer
    assert pf(h, None, 0, None, 0, None, None, 0, None, None, None, None, 0, None) == binding.PLE_ERR_INVALID_ARG
    # null pointers; a cache smaller than the hits (5 tokens x 4 heads = 20)
    assert pf(h, None, 5, 0x2000, 1, 0x3000, 0x4000, 20, 0x5000, 0x6000, 0x7000, 0x8000, 1 << 20, None) == \
        binding.PLE_ERR_INVALID_ARG
    assert pf(h, 0x1000, 5, 0x2000, 1, 0x3000, 0x4000, 19, 0x5000, 0x6000, 0x7000, 0x8000, 1 << 20, None) == \
        binding.PLE_ERR_INVALID_ARG
    # misaligned host table / cache / slots
    assert pf(h, 0x1000, 5, 0x2000, 1, 0x3008, 0x4000, 20, 0x5000, 0x6000, 0x7000, 0x8000, 1 << 20, None) == \
        binding.PLE_ERR_ALIGNMENT
    assert pf(h, 0x1000, 5, 0x2000, 1, 0x3000, 0x4008, 20, 0x5000, 0x6000, 0x7000, 0x8000, 1 << 20, None) == \
        binding.PLE_ERR_ALIGNMENT
    assert pf(h, 0x1000, 5, 0x2000, 1, 0x3000, 0x4000, 20, 0x5004, 0x6000, 0x7000, 0x8000, 1 << 20, None) == \
        binding.PLE_ERR_ALIGNMENT
    assert lib.ple_prefetch_workspace_bytes(h, 5) > 0 and lib.ple_prefetch_workspace_bytes(h, 0) == 0
    # gather and gradient from a cache: the usual checks, the cache size as the bound
    assert lib.ple_gather_cache(h, None, 0, None, 10, None, None) == 0
    assert lib.ple_gather_cache(h, 0x1000, 5, 0x2000, -1, 0x3000, None) == binding.PLE_ERR_INVALID_ARG
    assert lib.ple_gather_cache(h, 0x1000, 5, 0x2008, 10, 0x3000, None) == binding.PLE_ERR_ALIGNMENT
    assert lib.ple_grad_scatter_cache(h, 0x1000, 5, 0x2000, 1, 0x3000, 0, 0x4000, 1 << 20, None) == \
        binding.PLE_ERR_INVALID_ARG


def test_grad_halves_check_their_own_arguments():
    lib = ple.lib()
    p = _plan()
    h = p.handle
    need = lib.ple_grad_scatter_workspace_bytes(h, 5)
    assert lib.ple_grad_prepare(h, None, 0, None, 0, None) == 0
    assert lib.ple_grad_prepare(h, None, 5, 0x4000, need, None) == binding.PLE_ERR_INVALID_ARG
    assert lib.ple_grad_prepare(h, 0x1004, 5, 0x4000, need, None) == binding.PLE_ERR_ALIGNMENT
    assert lib.ple_grad_prepare(h, 0x1000, 5, 0x4000, need - 1, None) == binding.PLE_ERR_WORKSPACE
    assert lib.ple_grad_apply(h, 5, None, 1, 0x3000, 0x4000, need, None) == binding.PLE_ERR_INVALID_ARG
    assert lib.ple_grad_apply(h, 5, 0x2000, 9, 0x3000, 0x4000, need, None) == binding.PLE_ERR_INVALID_ARG
    assert lib.ple_grad_apply(h, 5, 0x2008, 1, 0x3000, 0x4000, need, None) == binding.PLE_ERR_ALIGNMENT
    assert lib.ple_grad_apply(h, 5, 0x2000, 1, 0x3000, 0x4100, need - 256, None) == binding.PLE_ERR_WORKSPACE


def test_wait_limit_setter_round_trips():
    """Host-only hook of include/ple_debug.h: the limit of the bounded waits."""
    default = ple.default_wait_limit_ns()
    assert default == 100_000_000
    prev = ple.set_wait_limit_ns(12345)
    try:
        assert prev == default
        assert ple.set_wait_limit_ns(0) == 12345
    finally:
        ple.set_wait_limit_ns(default)
    assert ple.set_wait_limit_ns(default) == default


def test_plans_hold_status_slots_until_destroyed():
    """Each plan holds one of 4095 status words; destroying plans returns
    them (host only)."""
    lib = ple.lib()
    plans = [_plan() for _ in range(50)]
    del plans
    import gc

    gc.collect()
    many = [_plan() for _ in range(4000)]  # fits only if the 50 above were returned
    assert len(many) == 4000
