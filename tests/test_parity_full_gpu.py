"""Full-size workloads on the GPU, in the configuration bench.py times.

Rows are compared with the oracle for every token.  Gathered values are
compared with the oracle on sampled hits (table rows regenerated on the host
by the input generator), and on every hit with torch's embedding gather of
the same device table (a library routine of the same definition).  The
gradient is compared with the oracle's per-row sums on every touched row,
bit for bit, and every untouched row must stay zero.
"""
import gc

import numpy as np
import pytest
import torch

import oracle
import synth
import hashed_gram_embedding_ple_b200 as ple
from gpu_util import dev_i32, dev_i64, device_grad, device_table, torch_to_values

pytestmark = pytest.mark.gpu


def _free():
    gc.collect()
    torch.cuda.empty_cache()


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def _oracle_rows(w):
    return oracle.rows(w.tokens, w.cu_seqlens, w.ngram_size, w.heads_per_ngram, w.eos_id, w.mults, w.primes,
                       w.offsets, threads=8)


def check_forward_full(w, dev, samples=8192):
    plan = ple.Plan.from_workload(w)
    table = device_table(w, dev)
    # input check: the device generator wrote the host generator's values
    rng = np.random.default_rng(7)
    probe = rng.integers(0, w.num_rows, 64)
    raw = table.view(torch.uint8) if table.dtype == torch.float8_e4m3fn else table
    np.testing.assert_array_equal(torch_to_values(raw[dev_i64(probe, dev)]), w.table_rows(probe))

    tok, cu = dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev)
    out, rows = ple.ple_lookup(plan, tok, cu, table, save_rows=True)
    assert ple.ple_status() == ple.PLE_OK
    ref_rows = _oracle_rows(w)
    got_rows = rows.cpu().numpy()
    np.testing.assert_array_equal(got_rows, ref_rows)
    # sampled hits against the oracle's gather of regenerated rows
    hits = rng.integers(0, w.num_hits, samples)
    flat = out.view(w.num_hits, w.head_dim)
    got = torch_to_values(flat[dev_i64(hits, dev)])
    sel = ref_rows.reshape(-1)[hits]
    uniq, inv = np.unique(sel, return_inverse=True)
    compact = w.table_rows(uniq)
    fp8 = w.table_dtype == synth.DTYPE_E4M3
    np.testing.assert_array_equal(got, oracle.gather_e4m3(inv, compact) if fp8 else oracle.gather(inv, compact))
    # every hit against torch's gather of the same table (and, for fp8 codes,
    # torch's own widening of the gathered codes; the generator draws no NaN code)
    if fp8:
        ref_all = table.view(torch.uint8).index_select(0, rows.view(-1)).view(torch.float8_e4m3fn)
        ref_all = ref_all.to(torch.bfloat16)
    else:
        ref_all = torch.nn.functional.embedding(rows.view(-1), table)
    assert torch.equal(_bits(out.view(-1, w.head_dim)), _bits(ref_all))
    del ref_all
    del table, out, flat
    _free()
    return ref_rows


def check_backward_full(w, dev, ref_rows):
    plan = ple.Plan.from_workload(w)
    N = ref_rows.size
    grad = device_grad(w, dev, N)
    rows = dev_i64(ref_rows.reshape(-1), dev)
    tg = torch.zeros(w.num_rows, w.head_dim, dtype=torch.float32, device=dev)
    ple.ple_grad_scatter(plan, rows, grad, tg)
    assert ple.ple_status() == ple.PLE_OK
    grad_host = torch_to_values(grad)
    np.testing.assert_array_equal(grad_host[:4], w.grad_rows(np.arange(4)))  # input check
    uniq, sums = oracle.grad_sums(ref_rows.reshape(-1), grad_host, threads=8)
    u_dev = dev_i64(uniq, dev)
    got = tg.index_select(0, u_dev).cpu().numpy()
    np.testing.assert_array_equal(got.view(np.uint32), sums.view(np.uint32))
    tg.index_fill_(0, u_dev, 0.0)
    assert not bool(tg.any())
    del grad, tg
    _free()


def test_single_layer_bf16_full(cuda_device):
    w = synth.single_layer_bf16(0)
    ref_rows = check_forward_full(w, cuda_device)
    check_backward_full(w, cuda_device, ref_rows)


def test_large_table_full(cuda_device):
    w = synth.large_table(0)
    assert w.table_bytes > 50e9
    check_forward_full(w, cuda_device)


def test_large_table_fp8_full(cuda_device):
    w = synth.large_table_fp8(0)
    assert w.table_bytes > 25e9
    check_forward_full(w, cuda_device)


def test_backward_stress_full(cuda_device):
    w = synth.backward_stress(0)
    plan = ple.Plan.from_workload(w)
    rows = ple.ple_hash(plan, dev_i64(w.tokens, cuda_device), dev_i32(w.cu_seqlens, cuda_device))
    ref_rows = _oracle_rows(w)
    np.testing.assert_array_equal(rows.cpu().numpy(), ref_rows)
    # heavy repetition: the hottest row is hit thousands of times
    counts = np.bincount(np.unique(ref_rows.ravel(), return_inverse=True)[1].ravel())
    assert counts.max() > 1000
    check_backward_full(w, cuda_device, ref_rows)


@pytest.mark.parametrize("kw", [
    dict(tokens=1 << 20, head_dim=32, ngram_size=2, ids="uniform", table_gb=16.0),
    dict(tokens=16384, head_dim=256, ngram_size=4, ids="zipf", table_gb=2.0),
    dict(tokens=131072, head_dim=128, ngram_size=3, ids="zipf", table_gb=80.0),
    dict(tokens=131072, head_dim=128, ngram_size=3, ids="zipf", table_gb=16.0, table_dtype=synth.DTYPE_E4M3),
])
def test_sweep_points(cuda_device, kw):
    w = synth.sweep_point(**kw)
    ref_rows = check_forward_full(w, cuda_device)
    if w.num_rows * w.head_dim * 4 <= 40e9:
        check_backward_full(w, cuda_device, ref_rows)
