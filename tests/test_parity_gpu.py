"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Rows, gathered values and the deterministic gradient must be bit-identical
to the oracle; the atomic gradient variant is held to a relative 1e-5.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import hashed_gram_embedding_ple_b200 as ple
from gpu_util import (custom_workload, dev_i32, dev_i64, host_grad, small_table, torch_to_values,
                      values_to_torch)

pytestmark = pytest.mark.gpu


def oracle_rows(w):
    return oracle.rows(w.tokens, w.cu_seqlens, w.ngram_size, w.heads_per_ngram, w.eos_id, w.mults, w.primes,
                       w.offsets)


def run_forward(w, dev):
    plan = ple.Plan.from_workload(w)
    tok, cu = dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev)
    host_table, table = small_table(w, dev)
    rows = ple.ple_hash(plan, tok, cu)
    out, rows_out = ple.ple_lookup(plan, tok, cu, table, save_rows=True)
    gathered = ple.ple_gather(plan, rows, table)
    assert ple.ple_status() == ple.PLE_OK
    return plan, host_table, rows.cpu().numpy(), rows_out.cpu().numpy(), torch_to_values(out), \
        torch_to_values(gathered)


def check_forward(w, dev):
    plan, host_table, rows, rows_out, out, gathered = run_forward(w, dev)
    ref_rows = oracle_rows(w)
    np.testing.assert_array_equal(rows, ref_rows)
    np.testing.assert_array_equal(rows_out, ref_rows)
    ref_out = oracle.gather(ref_rows, host_table)
    assert out.shape == ref_out.shape
    np.testing.assert_array_equal(out, ref_out)
    np.testing.assert_array_equal(gathered, ref_out)
    return ref_rows


def check_backward(w, dev, rows_np, prefill=None):
    plan = ple.Plan.from_workload(w)
    N = rows_np.size
    g_host = host_grad(w, N)
    g = values_to_torch(g_host, w.grad_dtype).to(dev)
    rows = dev_i64(rows_np.reshape(-1), dev)
    base = np.zeros((w.num_rows, w.head_dim), np.float32) if prefill is None else prefill.copy()
    tg = torch.from_numpy(base.copy()).to(dev)
    ple.ple_grad_scatter(plan, rows, g, tg)
    assert ple.ple_status() == ple.PLE_OK
    ref = oracle.grad_apply(rows_np.reshape(-1), g_host, base.copy())
    got = tg.cpu().numpy()
    np.testing.assert_array_equal(got.view(np.uint32), ref.view(np.uint32))
    # run to run: bit-identical again
    tg2 = torch.from_numpy(base.copy()).to(dev)
    ple.ple_grad_scatter(plan, rows, g, tg2)
    assert torch.equal(tg2.view(torch.int32), tg.view(torch.int32))
    # atomic variant: the same sums in an unspecified order.  Relative error
    # 1e-5 is measured against the magnitude sum |base| + sum |g| of each
    # element (the scale of any fp32 reordering error), since the sum itself
    # may cancel to near zero.
    tg3 = torch.from_numpy(base.copy()).to(dev)
    ple.ple_grad_scatter_atomic(plan, rows, g, tg3)
    torch.cuda.synchronize()
    g32 = torch.from_numpy(g_host.astype(np.float32) if w.grad_dtype == synth.DTYPE_F32 else
                           synth.bf16_bits_to_f32(g_host)).double()
    mag = torch.from_numpy(np.abs(base)).double().index_add_(0, torch.from_numpy(rows_np.reshape(-1)), g32.abs())
    err = np.abs(tg3.cpu().numpy().astype(np.float64) - ref.astype(np.float64))
    assert np.all(err <= 1e-5 * mag.numpy() + 1e-30)


# ---------------------------------------------------------------------------

def test_tiny_forward_backward(cuda_device):
    w = synth.tiny(0)
    rows = check_forward(w, cuda_device)
    check_backward(w, cuda_device, rows)


@pytest.mark.parametrize("n,G,D,dt", [
    (2, 1, 8, synth.DTYPE_BF16),     # 16-byte rows
    (3, 3, 48, synth.DTYPE_F32),     # 192-byte rows: 12 vectors, not a power of two
    (4, 2, 24, synth.DTYPE_BF16),    # 48-byte rows: 3 vectors
    (4, 5, 128, synth.DTYPE_BF16),
    (5, 4, 64, synth.DTYPE_F32),
    (8, 1, 256, synth.DTYPE_BF16),   # largest order
    (3, 32, 32, synth.DTYPE_F32),    # 64 heads
    (3, 32, 256, synth.DTYPE_F32),   # 64 heads of 1 KB rows: one token per warp, the generic fold at D = 256
])
def test_ragged_multi_tile(cuda_device, n, G, D, dt):
    rng = np.random.default_rng(100 + n * 10 + G)
    lens = [1, 0, 37, 5000 - 38 - 13, 13]  # several tiles, a ragged tail, an empty and a 1-token sequence
    T = sum(lens)
    tok = rng.integers(0, 50, T)  # small vocabulary: many repeats and many EOS (id 0)
    mults = synth.signed_mults(n, rng)
    primes = synth.consecutive_primes(int(rng.integers(50, 400)), (n - 1) * G)
    w = custom_workload("ragged", tok, synth.cu_seqlens_from_lengths(lens), n, G, 0, mults, primes, D, dt, dt,
                        seed=n)
    rows = check_forward(w, cuda_device)
    check_backward(w, cuda_device, rows)


def test_production_constants_forward(cuda_device):
    from conftest import read_golden_blocks

    _, g = read_golden_blocks("production_constants.txt")
    primes = synth.consecutive_primes(20_000_000, 16)
    rng = np.random.default_rng(1)
    T = 3000
    tok = rng.integers(0, 248_320, T)
    tok[rng.random(T) < 0.02] = g["eos_token_id"][0]
    w = custom_workload("prod", tok, [0, 1234, T], 3, 8, g["eos_token_id"][0], g["multipliers"], primes, 8,
                        synth.DTYPE_BF16)
    plan = ple.Plan.from_workload(w)
    rows = ple.ple_hash(plan, dev_i64(w.tokens, cuda_device), dev_i32(w.cu_seqlens, cuda_device))
    np.testing.assert_array_equal(rows.cpu().numpy(), oracle_rows(w))


def test_edge_cases(cuda_device):
    dev = cuda_device
    rng = np.random.default_rng(3)
    mults = [2 ** 63 - 1, -(2 ** 63), 12345]
    # all EOS; single token; alternating EOS; many 1-token sequences
    cases = [
        (np.zeros(70, np.int64), [0, 70]),
        (np.array([5], np.int64), [0, 1]),
        (np.tile([0, 7], 40), [0, 80]),
        (rng.integers(0, 5, 100), list(range(0, 101))),
        (rng.integers(0, 5, 64), [0, 0, 0, 32, 32, 64, 64]),
    ]
    for k, (tok, cu) in enumerate(cases):
        w = custom_workload(f"edge{k}", tok, cu, 3, 2, 0, mults, [5, 7, 11, 13], 8, synth.DTYPE_F32)
        rows = check_forward(w, dev)
        check_backward(w, dev, rows)


def test_empty_inputs(cuda_device):
    w = synth.tiny(0)
    plan = ple.Plan.from_workload(w)
    tok = torch.empty(0, dtype=torch.int64, device=cuda_device)
    cu = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    _, table = small_table(w, cuda_device)
    assert ple.ple_hash(plan, tok, cu).shape == (0, 4)
    assert ple.ple_lookup(plan, tok, cu, table).shape == (0, 4, 32)
    tg = torch.zeros(w.num_rows, w.head_dim, device=cuda_device)
    ple.ple_grad_scatter(plan, tok, torch.empty(0, 32, device=cuda_device), tg)
    assert ple.ple_status() == ple.PLE_OK and not tg.any()


def test_gradient_chunk_boundaries(cuda_device):
    """Rows hit exactly 1, 31, 32, 33, 64, 65, 1000 and 5000 times, interleaved."""
    rng = np.random.default_rng(5)
    counts = {3: 1, 10: 31, 11: 32, 12: 33, 20: 64, 21: 65, 30: 1000, 31: 5000}
    rows = np.concatenate([np.full(c, r) for r, c in counts.items()] + [rng.integers(0, 40, 3000)])
    rows = rng.permutation(rows)
    w = custom_workload("chunks", np.zeros(1, np.int64), [0, 1], 2, 1, 0, [1, 1], [41], 64, synth.DTYPE_F32,
                        synth.DTYPE_BF16)
    prefill = synth.dense_values(9, 41 * 64, 0.5, synth.DTYPE_F32).reshape(41, 64)
    check_backward(w, cuda_device, rows, prefill=prefill)


@pytest.mark.parametrize("D,gdt,N", [(128, synth.DTYPE_BF16, 300_001), (40, synth.DTYPE_F32, 300_001),
                                     (64, synth.DTYPE_BF16, 512 * 32 + 50), (64, synth.DTYPE_BF16, 512 * 32 + 51)])
def test_gradient_every_hit_on_one_row(cuda_device, D, gdt, N):
    """The degenerate input of identical tokens: (nearly) every hit of the
    call lands on one row, one run of up to 300,001 hits (9,376 chunk sums
    folded in order by finish_long_runs_kernel), plus 50 hits on other rows;
    the run of exactly 512 chunks stays inside the fold, 513 chunks do not."""
    rng = np.random.default_rng(D + N)
    rows = np.full(N, 7, np.int64)
    rows[rng.choice(N, 50, replace=False)] = rng.integers(8, 40, 50)  # the hot row keeps exactly N - 50 hits
    w = custom_workload("one_row", np.zeros(1, np.int64), [0, 1], 2, 1, 0, [1, 1], [41], D, synth.DTYPE_F32, gdt)
    check_backward(w, cuda_device, rows)


@pytest.mark.parametrize("D,gdt", [(32, synth.DTYPE_F32), (64, synth.DTYPE_BF16), (128, synth.DTYPE_BF16),
                                   (256, synth.DTYPE_F32), (40, synth.DTYPE_BF16), (200, synth.DTYPE_F32)])
def test_gradient_many_tiles(cuda_device, D, gdt):
    """Zipf-heavy rows over several sort tiles and a ragged tail."""
    rng = np.random.default_rng(D)
    R = 70_001
    N = 3 * 4096 + 1234
    rows = synth.zipf_ids(N, 1.3, R, rng)
    w = custom_workload("gtiles", np.zeros(1, np.int64), [0, 1], 2, 1, 0, [1, 1], [R], D, synth.DTYPE_F32, gdt)
    check_backward(w, cuda_device, rows)


@pytest.mark.parametrize("N", [3 * 2**17 - 1, 3 * 2**17 + 777, 37 * 2**15 - 1, 37 * 2**15 + 4097])
def test_gradient_both_sort_tile_sizes(cuda_device, N):
    """Just below and above the key counts at which the sort passes switch
    from 2048-key to 4096-key tiles and from 4096-key to 8192-key tiles
    (ragged last tile on both sides)."""
    rng = np.random.default_rng(N)
    R = 1_000_003
    rows = synth.zipf_ids(N, 1.2, R, rng)
    w = custom_workload("gswitch", np.zeros(1, np.int64), [0, 1], 2, 1, 0, [1, 1], [R], 16, synth.DTYPE_F32,
                        synth.DTYPE_BF16)
    check_backward(w, cuda_device, rows)


# fp32 values at the edge of the final add: signed zeros, subnormals, the
# smallest normal, and values around 2^-100 (the reduction / exact-add switch)
_SPECIAL_F32 = np.array([0.0, -0.0, 1e-45, -1e-45, 1e-40, -1e-40, 3e-39, -5.877e-39, 2.0 ** -126, -(2.0 ** -127),
                         2.0 ** -100, -(2.0 ** -101), 1.0, -1.5], np.float32)
# bf16 bit patterns: +-0, the smallest and largest subnormal, the smallest normal, ordinary values
_SPECIAL_BF16 = np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x007F, 0x807F, 0x0080, 0x8080, 0x0040, 0x3F80, 0xBFC0],
                         np.uint16)


def _special_grad(rng, n, D, gdt, modes):
    """Per hit row: mode 0 random specials, 1 all -0, 2 all subnormal, 3 all +0."""
    if gdt == synth.DTYPE_F32:
        pool, neg0, pos0, sub = _SPECIAL_F32, np.float32(-0.0), np.float32(0.0), _SPECIAL_F32[2:8]
    else:
        pool, neg0, pos0, sub = _SPECIAL_BF16, np.uint16(0x8000), np.uint16(0), _SPECIAL_BF16[2:6]
    g = pool[rng.integers(0, len(pool), (n, D))]
    g[modes == 1] = neg0
    g[modes == 3] = pos0
    g[modes == 2] = sub[rng.integers(0, len(sub), (int((modes == 2).sum()), D))]
    return g


@pytest.mark.parametrize("D,gdt", [(32, synth.DTYPE_F32), (64, synth.DTYPE_BF16), (128, synth.DTYPE_BF16),
                                   (64, synth.DTYPE_F32), (40, synth.DTYPE_BF16), (200, synth.DTYPE_F32)])
def test_gradient_signed_zero_and_subnormal(cuda_device, D, gdt):
    """The final add table_grad + S_r is the IEEE fp32 add: -0 + -0 stays -0,
    subnormal sums and subnormal prefills are kept.  Rows hit once (whole-run
    add), 2..33 times, 64, 65 and 1000 times (chunk slots and the run's
    second level), with all-(-0), all-(+0), all-subnormal and mixed rows, on
    the wide folds (D = 32, 64, 128) and the generic fold (D = 40, 200)."""
    dev = cuda_device
    rng = np.random.default_rng(4000 + D + gdt)
    counts = [1] * 120 + [2] * 40 + [31, 32, 33] * 6 + [64, 65, 1000]
    R = len(counts) + 17  # rows never hit keep their prefill
    rows = np.concatenate([np.full(c, r, np.int64) for r, c in enumerate(counts)])
    row_mode = rng.integers(0, 4, R)
    perm = rng.permutation(rows.size)
    rows = rows[perm]
    g_host = _special_grad(rng, rows.size, D, gdt, row_mode[rows])
    prefill = _SPECIAL_F32[rng.integers(0, len(_SPECIAL_F32), (R, D))].copy()
    prefill[row_mode == 1] = np.float32(-0.0)
    w = custom_workload("subn", np.zeros(1, np.int64), [0, 1], 2, 1, 0, [1, 1], [R], D, synth.DTYPE_F32, gdt)
    plan = ple.Plan.from_workload(w)
    g = values_to_torch(g_host, gdt).to(dev)
    ref = oracle.grad_apply(rows, g_host, prefill.copy())
    assert np.any(np.signbit(ref) & (ref == 0)), "the case must hold -0 results"
    assert np.any((ref != 0) & (np.abs(ref) < np.float32(2.0 ** -126))), "and subnormal results"
    for entry in ("scatter", "noalloc"):
        tg = torch.from_numpy(prefill.copy()).to(dev)
        if entry == "scatter":
            ple.ple_grad_scatter(plan, dev_i64(rows, dev), g, tg)
        else:
            ple.ple_grad_scatter_noalloc(plan, dev_i64(rows, dev), g, tg)
        assert ple.ple_status() == ple.PLE_OK
        np.testing.assert_array_equal(tg.cpu().numpy().view(np.uint32), ref.view(np.uint32), err_msg=entry)


def test_bad_rows_flagged(cuda_device):
    dev = cuda_device
    w = synth.tiny(0)
    plan = ple.Plan.from_workload(w)
    host_table, table = small_table(w, dev)
    rows_np = np.array([5, -1, 24591, 24592, 2 ** 40, 7], np.int64)
    out = ple.ple_gather(plan, dev_i64(rows_np, dev), table)
    assert ple.ple_status() == ple.PLE_ERR_BAD_ROW
    assert ple.ple_status() == ple.PLE_OK  # cleared
    o = out.cpu().numpy()
    np.testing.assert_array_equal(o[[0, 2, 5]], host_table[[5, 24591, 7]])
    assert not o[[1, 3, 4]].any()
    # gradient: bad hits dropped, the rest exact
    g_host = host_grad(w, len(rows_np))
    tg = torch.zeros(w.num_rows, w.head_dim, device=dev)
    ple.ple_grad_scatter(plan, dev_i64(rows_np, dev), values_to_torch(g_host, w.grad_dtype).to(dev), tg)
    assert ple.ple_status() == ple.PLE_ERR_BAD_ROW
    good = np.array([0, 2, 5])
    ref = oracle.grad_apply(rows_np[good], g_host[good], np.zeros((w.num_rows, w.head_dim), np.float32))
    np.testing.assert_array_equal(tg.cpu().numpy(), ref)


def test_malformed_seqlens_flagged(cuda_device):
    dev = cuda_device
    w = synth.tiny(0)
    plan = ple.Plan.from_workload(w)
    tok = dev_i64(w.tokens, dev)
    for bad in ([0, 200, 100, 256], [1, 100, 256], [0, 100, 250]):
        rows = ple.ple_hash(plan, tok, dev_i32(bad, dev))
        assert ple.ple_status() == ple.PLE_ERR_BAD_SEQLENS
        r = rows.cpu().numpy()
        assert np.all(r >= w.offsets) and np.all(r < w.offsets + w.primes)


def test_library_loaded_from_tree(cuda_device):
    import os

    ple.lib()
    maps = open("/proc/self/maps").read()
    assert os.path.realpath(ple.binding.LIB_PATH) in maps


@pytest.mark.parametrize("row_len,B,start,end", [(256, 1, 0, 256), (256, 1, 100, 180), (1000, 4, 333, 777),
                                                 (64, 8, 0, 1), (64, 8, 63, 64), (300, 3, 17, 17)])
def test_global_slice_lookup(cuda_device, row_len, B, start, end):
    dev = cuda_device
    rng = np.random.default_rng(row_len + start)
    T = row_len * B
    tok = rng.integers(0, 60, T)
    tok[rng.random(T) < 0.05] = 0
    # packed segments inside every row (a boundary at each row start, and one more per row)
    cuts = sorted(set([b * row_len for b in range(B + 1)] + [b * row_len + row_len // 3 for b in range(B)]))
    w = custom_workload("slice", tok, cuts, 4, 3, 0, synth.signed_mults(4, rng), synth.consecutive_primes(331, 9),
                        40, synth.DTYPE_BF16)
    plan = ple.Plan.from_workload(w)
    host_table, table = small_table(w, dev)
    out, rows = ple.ple_lookup_slice(plan, dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev), row_len, start, end,
                                     table, save_rows=True)
    assert ple.ple_status() == ple.PLE_OK
    ref_vals, ref_rows = oracle.lookup_slice(w.tokens, w.cu_seqlens, w.ngram_size, w.heads_per_ngram, w.eos_id,
                                             w.mults, w.primes, w.offsets, host_table, row_len, start, end)
    assert out.shape == (B, end - start, w.num_heads, w.head_dim)
    np.testing.assert_array_equal(rows.cpu().numpy(), ref_rows)
    np.testing.assert_array_equal(torch_to_values(out), ref_vals)


def test_prepare_then_apply_equals_scatter(cuda_device):
    """The two halves of the gradient, the prepare on a second stream beside
    other work, give the same bits as ple_grad_scatter."""
    dev = cuda_device
    rng = np.random.default_rng(21)
    lens = [3, 700, 0, 4000, 1]
    tok = rng.integers(0, 40, sum(lens))  # heavy repeats: long runs
    w = custom_workload("split", tok, synth.cu_seqlens_from_lengths(lens), 3, 4, 0, synth.signed_mults(3, rng),
                        synth.consecutive_primes(97, 8), 64, synth.DTYPE_BF16, synth.DTYPE_BF16, seed=4)
    plan = ple.Plan.from_workload(w)
    tok_d, cu_d = dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev)
    g = values_to_torch(host_grad(w), w.grad_dtype).to(dev)
    N = w.num_hits
    ref = torch.zeros(w.num_rows, w.head_dim, device=dev)
    ple.ple_grad_scatter(plan, ple.ple_hash(plan, tok_d, cu_d).view(-1), g, ref)
    side = torch.cuda.Stream(dev)
    ws = ple.alloc_workspace(plan, N, dev)
    with torch.cuda.stream(side):
        rows = ple.ple_hash(plan, tok_d, cu_d)
        ple.ple_grad_prepare(plan, rows.view(-1), ws)
    _, table = small_table(w, dev)
    out = ple.ple_lookup(plan, tok_d, cu_d, table)  # the forward, concurrently on the main stream
    torch.cuda.current_stream(dev).wait_stream(side)
    tg = torch.zeros(w.num_rows, w.head_dim, device=dev)
    ple.ple_grad_apply(plan, N, g, tg, ws)
    assert ple.ple_status() == ple.PLE_OK
    assert out.shape == (w.num_tokens, w.num_heads, w.head_dim)
    assert torch.equal(tg.view(torch.int32), ref.view(torch.int32))


def _poison(ws, fill, seed=0):
    if fill == "random":
        g = torch.Generator(device=ws.device).manual_seed(seed)
        ws.copy_(torch.randint(0, 256, ws.shape, dtype=torch.uint8, device=ws.device, generator=g))
    else:
        ws.fill_(fill)


@pytest.mark.parametrize("fill", [0x00, 0xFF, "random"])
@pytest.mark.parametrize("N", [3 * 4096 + 1234, 3 * 2**17 + 5, 37 * 2**15 + 999])
def test_gradient_workspace_contents_do_not_matter(cuda_device, fill, N):
    """The caller's workspace may hold anything (a reused buffer, bytes left
    by another call): every word the gradient needs cleared (digit totals,
    tile tickets, the abort word, look-back rows, run counters) is cleared by
    the call itself.  All three sort tile sizes; ple_grad_scatter and the
    prepare / apply halves, against the oracle."""
    dev = cuda_device
    rng = np.random.default_rng(N)
    R = 1_000_003
    rows = synth.zipf_ids(N, 1.2, R, rng)
    w = custom_workload("poison", np.zeros(1, np.int64), [0, 1], 2, 1, 0, [1, 1], [R], 16, synth.DTYPE_F32,
                        synth.DTYPE_BF16, seed=N % 97)
    plan = ple.Plan.from_workload(w)
    g_host = host_grad(w, N)
    g = values_to_torch(g_host, w.grad_dtype).to(dev)
    rows_d = dev_i64(rows, dev)
    ref = oracle.grad_apply(rows, g_host, np.zeros((R, 16), np.float32))
    ws = ple.alloc_workspace(plan, N, dev)
    _poison(ws, fill, seed=1)
    tg = torch.zeros(R, 16, device=dev)
    ple.ple_grad_scatter(plan, rows_d, g, tg, workspace=ws)
    assert ple.ple_status(dev, plan=plan) == ple.PLE_OK
    np.testing.assert_array_equal(tg.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    _poison(ws, fill, seed=2)
    tg.zero_()
    ple.ple_grad_prepare(plan, rows_d, ws)
    ple.ple_grad_apply(plan, N, g, tg, ws)
    assert ple.ple_status(dev, plan=plan) == ple.PLE_OK
    np.testing.assert_array_equal(tg.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("fill", [0xFF, "random"])
def test_prefetch_and_conv_workspace_contents_do_not_matter(cuda_device, fill):
    """ple_prefetch and ple_conv_backward give the same bits with a poisoned
    workspace as with a zeroed one."""
    dev = cuda_device
    rng = np.random.default_rng(77)
    lens = [300, 0, 4000, 1, 2500]
    tok = rng.integers(0, 200, sum(lens))
    w = custom_workload("pf_poison", tok, synth.cu_seqlens_from_lengths(lens), 3, 4, 0, synth.signed_mults(3, rng),
                        synth.consecutive_primes(5003, 8), 32, synth.DTYPE_BF16, synth.DTYPE_BF16)
    plan = ple.Plan.from_workload(w)
    host_table, _ = small_table(w, dev)
    pinned = values_to_torch(host_table, w.table_dtype).pin_memory()
    tok_d, cu_d = dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev)
    outs = []
    for poison in (False, True):
        buf = ple.Prefetched(plan, w.num_tokens, dev)
        if poison:
            _poison(buf.workspace, fill, seed=3)
        else:
            buf.workspace.zero_()
        ple.ple_prefetch(plan, tok_d, cu_d, pinned, buf)
        assert ple.ple_status(dev, plan=plan) == ple.PLE_OK
        U = int(buf.num_unique.item())
        outs.append((U, buf.slots.clone(), buf.uniq_rows[:U].clone(), buf.cache[:U].clone()))
    assert outs[0][0] == outs[1][0]
    for a, b in zip(outs[0][1:], outs[1][1:]):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    # conv backward: partial-sum workspace
    T, C, K, d = sum(lens), 64, 4, 3
    x = torch.from_numpy(rng.standard_normal((T, C)).astype(np.float32)).to(dev)
    dy = torch.from_numpy(rng.standard_normal((T, C)).astype(np.float32)).to(dev)
    wt = torch.from_numpy(rng.standard_normal((C, K)).astype(np.float32)).to(dev)
    cu = dev_i32(synth.cu_seqlens_from_lengths(lens), dev)
    res = []
    for poison in (False, True):
        ws = torch.empty(ple.conv_workspace_bytes(T, C, K), dtype=torch.uint8, device=dev)
        if poison:
            _poison(ws, fill, seed=4)
        else:
            ws.zero_()
        dw, db = torch.zeros(C, K, device=dev), torch.zeros(C, device=dev)
        dx, _, _ = ple.conv_backward(dy, x, cu, wt, d, dweight=dw, dbias=db, workspace=ws)
        res.append((dx, dw, db))
    assert ple.ple_status(dev) == ple.PLE_OK
    for a, b in zip(*res):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
