"""Host-memory tier through the C ABI against the oracle: the table in pinned
host memory, the distinct rows of a batch prefetched into a device cache,
the lookup gathered from the cache and the gradient summed per cache row.

Everything here is exact: the distinct rows and slots are integers, the cache
and the lookup are copies (the fp8 widening is exact), and the cache gradient
of row u is the same fixed-order sum as the table gradient of uniq_rows[u]."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import hashed_gram_embedding_ple_b200 as ple
from gpu_util import custom_workload, dev_i32, dev_i64, host_grad, torch_to_values, values_to_torch

pytestmark = pytest.mark.gpu


def _pinned_table(w):
    v = synth.dense_values(w.table_seed, w.num_rows * w.head_dim, w.table_sigma, w.table_dtype)
    host = v.reshape(w.num_rows, w.head_dim)
    return host, values_to_torch(host, w.table_dtype).pin_memory()


def check_prefetch(w, dev, grad=True):
    plan = ple.Plan.from_workload(w)
    host, table = _pinned_table(w)
    tok, cu = dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev)
    side = torch.cuda.Stream(dev)
    with torch.cuda.stream(side):  # the prefetch on its own stream, as a pipeline would run it
        buf = ple.ple_prefetch(plan, tok, cu, table)
    torch.cuda.current_stream(dev).wait_stream(side)
    out = ple.ple_gather_cache(plan, buf)
    assert ple.ple_status() == ple.PLE_OK
    rows = oracle.rows(w.tokens, w.cu_seqlens, w.ngram_size, w.heads_per_ngram, w.eos_id, w.mults, w.primes, w.offsets)
    uniq = np.unique(rows)
    U = int(buf.num_unique.item())
    assert U == uniq.size
    got_uniq = buf.uniq_rows[:U].cpu().numpy()
    np.testing.assert_array_equal(got_uniq, uniq)
    slots = buf.slots.cpu().numpy()
    assert slots.min() >= 0 and slots.max() < U
    np.testing.assert_array_equal(got_uniq[slots], rows)
    cache_rows = torch_to_values(buf.cache[:U])
    np.testing.assert_array_equal(cache_rows, host[uniq])
    ref = oracle.gather_e4m3(rows, host) if w.table_dtype == synth.DTYPE_E4M3 else oracle.gather(rows, host)
    np.testing.assert_array_equal(torch_to_values(out), ref)
    if grad:
        g_host = host_grad(w, rows.size)
        g = values_to_torch(g_host, w.grad_dtype).to(dev)
        cg = ple.ple_grad_scatter_cache(plan, buf, g)
        assert ple.ple_status() == ple.PLE_OK
        u_rows, sums = oracle.grad_sums(rows.reshape(-1), g_host)
        np.testing.assert_array_equal(u_rows, uniq)
        got = cg[:U].cpu().numpy()
        np.testing.assert_array_equal(got.view(np.uint32), sums.view(np.uint32))
        assert not bool(cg[U:].any())
    return buf


@pytest.mark.parametrize("n,G,D,dt", [
    (3, 2, 64, synth.DTYPE_BF16),
    (4, 3, 48, synth.DTYPE_F32),
    (2, 8, 16, synth.DTYPE_BF16),
    (3, 2, 128, synth.DTYPE_E4M3),
])
def test_prefetch_ragged(cuda_device, n, G, D, dt):
    rng = np.random.default_rng(n * 100 + G)
    lens = [1, 0, 37, 5000 - 38 - 13, 13]
    tok = rng.integers(0, 60, sum(lens))  # small vocabulary: many repeated rows
    w = custom_workload("host tier", tok, synth.cu_seqlens_from_lengths(lens), n, G, 0, synth.signed_mults(n, rng),
                        synth.consecutive_primes(int(rng.integers(50, 400)), (n - 1) * G), D, dt, synth.DTYPE_BF16,
                        seed=n + 7)
    check_prefetch(w, cuda_device, grad=dt != synth.DTYPE_E4M3)


def test_prefetch_tiny_and_empty(cuda_device):
    dev = cuda_device
    check_prefetch(synth.tiny(0), dev)
    w = synth.tiny(0)
    plan = ple.Plan.from_workload(w)
    _, table = _pinned_table(w)
    buf = ple.ple_prefetch(plan, torch.empty(0, dtype=torch.int64, device=dev),
                           torch.zeros(2, dtype=torch.int32, device=dev), table)
    assert int(buf.num_unique.item()) == 0


def test_prefetch_rejects_pageable_host_memory(cuda_device):
    dev = cuda_device
    w = synth.tiny(0)
    plan = ple.Plan.from_workload(w)
    buf = ple.Prefetched(plan, w.num_tokens, dev)
    pageable = np.zeros((w.num_rows, w.head_dim), np.float32)
    tok, cu = dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev)
    rc = ple.lib().ple_prefetch(plan.handle, tok.data_ptr(), w.num_tokens, cu.data_ptr(), len(w.cu_seqlens) - 1,
                                pageable.ctypes.data, buf.cache.data_ptr(), buf.cache_rows, buf.slots.data_ptr(),
                                buf.uniq_rows.data_ptr(), buf.num_unique.data_ptr(), buf.workspace.data_ptr(),
                                buf.workspace.numel(), None)
    assert rc == ple.binding.PLE_ERR_INVALID_ARG


def test_prefetch_single_layer_full(cuda_device):
    """The bench's single-layer workload with its 2.05 GB table pinned on the host."""
    from synth import gpu as sgpu

    dev = cuda_device
    w = synth.single_layer_bf16(0)
    plan = ple.Plan.from_workload(w)
    dtable = torch.empty(w.num_rows, w.head_dim, dtype=torch.bfloat16, device=dev)
    sgpu.fill_(dtable, w.table_seed, w.table_sigma)
    table = torch.empty(w.num_rows, w.head_dim, dtype=torch.bfloat16, pin_memory=True)
    table.copy_(dtable)
    tok, cu = dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev)
    buf = ple.ple_prefetch(plan, tok, cu, table)
    out = ple.ple_gather_cache(plan, buf)
    ref, rows = ple.ple_lookup(plan, tok, cu, dtable, save_rows=True)
    assert ple.ple_status() == ple.PLE_OK
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    U = int(buf.num_unique.item())
    assert U == int(torch.unique(rows).numel())
    assert torch.equal(buf.uniq_rows[:U][buf.slots.view(-1)], rows.view(-1))
    # the cache gradient equals the table gradient's touched rows, bit for bit
    g = torch.empty(w.num_hits, w.head_dim, dtype=torch.bfloat16, device=dev)
    sgpu.fill_(g, w.grad_seed, w.grad_sigma)
    cg = ple.ple_grad_scatter_cache(plan, buf, g)
    tg = torch.zeros(w.num_rows, w.head_dim, device=dev)
    ple.ple_grad_scatter(plan, rows.view(-1), g, tg)
    assert torch.equal(cg[:U].view(torch.int32), tg[buf.uniq_rows[:U]].view(torch.int32))
