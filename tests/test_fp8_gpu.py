"""fp8 E4M3 tables through the C ABI against the oracle.

The lookup and the gather of an E4M3 table write bf16.  Every finite code
widens exactly and the two NaN codes (S.1111.111) give the quiet bf16 NaN of
their sign, so every output must equal the oracle's bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import hashed_gram_embedding_ple_b200 as ple
from gpu_util import custom_workload, dev_i32, dev_i64, host_grad, small_table, torch_to_values, values_to_torch

pytestmark = pytest.mark.gpu


def assert_widened(got, ref, codes):
    """got, ref: bf16 bit patterns; codes: the E4M3 codes they come from."""
    assert got.shape == ref.shape == codes.shape
    np.testing.assert_array_equal(got, ref)
    nan = (codes & 0x7F) == 0x7F
    assert nan.any() and np.all(np.isnan(synth.bf16_bits_to_f32(got[nan])))


def gather_plan(R, D):
    return ple.Plan(2, 1, 0, [1, 1], [R], [0], R, D, torch.float8_e4m3fn)


@pytest.mark.parametrize("D", [16, 48, 256])
def test_every_code_widens(cuda_device, D):
    dev = cuda_device
    rng = np.random.default_rng(D)
    # all 256 codes, each at several columns of several rows
    R = 64
    codes = np.concatenate([rng.permutation(256).astype(np.uint8) for _ in range(R * D // 256 + 1)])[:R * D]
    codes = codes.reshape(R, D)
    table = values_to_torch(codes, synth.DTYPE_E4M3).to(dev)
    rows_np = np.concatenate([np.arange(R), rng.integers(0, R, 3000)])
    out = ple.ple_gather(gather_plan(R, D), dev_i64(rows_np, dev), table)
    assert ple.ple_status() == ple.PLE_OK
    assert out.dtype == torch.bfloat16 and out.shape == (len(rows_np), D)
    got = torch_to_values(out)
    assert_widened(got, oracle.gather_e4m3(rows_np, codes), codes[rows_np])
    # torch's own E4M3 -> bf16 conversion agrees on every finite code
    finite = (codes[rows_np] & 0x7F) != 0x7F
    ref_t = torch_to_values(table.view(torch.uint8).index_select(0, dev_i64(rows_np, dev))
                            .view(torch.float8_e4m3fn).to(torch.bfloat16))
    np.testing.assert_array_equal(got[finite], ref_t[finite])


@pytest.mark.parametrize("n,G,D", [
    (2, 1, 16),     # 16-byte code rows
    (3, 3, 48),     # 3 vectors per row: not a power of two
    (4, 5, 128),
    (8, 1, 1024),   # 64 vectors per row, largest order
    (3, 2, 1040),   # 65 vectors per row
    (3, 32, 32),    # 64 heads
])
def test_fp8_lookup_ragged_multi_tile(cuda_device, n, G, D):
    dev = cuda_device
    rng = np.random.default_rng(300 + n * 10 + G)
    lens = [1, 0, 37, 5000 - 38 - 13, 13]
    T = sum(lens)
    tok = rng.integers(0, 50, T)
    mults = synth.signed_mults(n, rng)
    primes = synth.consecutive_primes(int(rng.integers(50, 400)), (n - 1) * G)
    w = custom_workload("fp8", tok, synth.cu_seqlens_from_lengths(lens), n, G, 0, mults, primes, D,
                        synth.DTYPE_E4M3, synth.DTYPE_BF16, seed=n + 40)
    plan = ple.Plan.from_workload(w)
    host_table, table = small_table(w, dev)
    assert host_table.dtype == np.uint8 and table.dtype == torch.float8_e4m3fn
    tok_d, cu_d = dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev)
    out, rows = ple.ple_lookup(plan, tok_d, cu_d, table, save_rows=True)
    gathered = ple.ple_gather(plan, rows, table)
    assert ple.ple_status() == ple.PLE_OK
    ref_rows = oracle.rows(w.tokens, w.cu_seqlens, n, G, 0, w.mults, w.primes, w.offsets)
    np.testing.assert_array_equal(rows.cpu().numpy(), ref_rows)
    ref = oracle.gather_e4m3(ref_rows, host_table)
    assert out.dtype == torch.bfloat16 and out.shape == (T, w.num_heads, D)
    np.testing.assert_array_equal(torch_to_values(out), ref)
    np.testing.assert_array_equal(torch_to_values(gathered), ref)
    # the backward of a lookup from an fp8 table: fp32 gradient of the rows,
    # the same deterministic sums as for any other table type
    g_host = host_grad(w, ref_rows.size)
    g = values_to_torch(g_host, w.grad_dtype).to(dev)
    tg = torch.zeros(w.num_rows, D, dtype=torch.float32, device=dev)
    if D > 256:  # the gradient's documented head_dim limit
        with pytest.raises(ple.PleError) as ei:
            ple.ple_grad_scatter(plan, rows.view(-1), g, tg)
        assert ei.value.status == ple.binding.PLE_ERR_UNSUPPORTED
        return
    ple.ple_grad_scatter(plan, rows.view(-1), g, tg)
    assert ple.ple_status() == ple.PLE_OK
    ref_g = oracle.grad_apply(ref_rows.reshape(-1), g_host, np.zeros((w.num_rows, D), np.float32))
    np.testing.assert_array_equal(tg.cpu().numpy().view(np.uint32), ref_g.view(np.uint32))


@pytest.mark.parametrize("row_len,B,start,end", [(256, 1, 100, 180), (1000, 4, 333, 777), (64, 8, 63, 64)])
def test_fp8_global_slice(cuda_device, row_len, B, start, end):
    dev = cuda_device
    rng = np.random.default_rng(row_len + start + 7)
    T = row_len * B
    tok = rng.integers(0, 60, T)
    tok[rng.random(T) < 0.05] = 0
    cuts = sorted(set([b * row_len for b in range(B + 1)] + [b * row_len + row_len // 3 for b in range(B)]))
    w = custom_workload("fp8 slice", tok, cuts, 4, 3, 0, synth.signed_mults(4, rng), synth.consecutive_primes(331, 9),
                        64, synth.DTYPE_E4M3)
    plan = ple.Plan.from_workload(w)
    host_table, table = small_table(w, dev)
    out, rows = ple.ple_lookup_slice(plan, dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev), row_len, start, end,
                                     table, save_rows=True)
    assert ple.ple_status() == ple.PLE_OK
    all_rows = oracle.rows(w.tokens, w.cu_seqlens, 4, 3, 0, w.mults, w.primes, w.offsets)
    pos = oracle.slice_positions(T, row_len, start, end)
    ref_rows = all_rows[pos].reshape(B, end - start, w.num_heads)
    np.testing.assert_array_equal(rows.cpu().numpy(), ref_rows)
    assert out.dtype == torch.bfloat16 and out.shape == (B, end - start, w.num_heads, 64)
    np.testing.assert_array_equal(torch_to_values(out), oracle.gather_e4m3(ref_rows, host_table))

